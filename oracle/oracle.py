"""fp64 CPU oracle for the Kimi Delta Attention recurrence -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It wraps ``kda_oracle.c`` (plain C, fp64,
one serial token loop per (sequence, head)) through ctypes, and shares nothing
with the CUDA library in ``gated_delta_rule_108_b200``.

The recurrence (daiw.net "Kimi Delta Attention", section "KDA 的更新式"):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = d_k^{-1/2} S_t^T q_t,        alpha_t = exp(log_alpha_t),

evaluated in the step order of news.bugfactory.tech/news/3610 (forget per
channel, predict on the decayed state, correct, write, read).  Inputs are taken
as given (already rounded to the caller's dtype) and upcast exactly to fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile kda_oracle.c into oracle/libkda_oracle.so with gcc -fopenmp."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_kda_forward.restype = ctypes.c_int
    lib.oracle_kda_forward.argtypes = [
        dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp,
    ]
    lib.oracle_kda_backward.restype = ctypes.c_int
    lib.oracle_kda_backward.argtypes = [
        dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp,
        dp, dp, dp, dp, dp, dp,
    ]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build_oracle())
    return _lib


def _f64(x) -> np.ndarray:
    """Exact upcast to a contiguous fp64 numpy array (torch or numpy input)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def _seqlens(cu_seqlens, B, T):
    if cu_seqlens is None:
        return np.arange(B + 1, dtype=np.int64) * T
    if B != 1:
        raise ValueError("cu_seqlens requires B == 1")
    if hasattr(cu_seqlens, "detach"):
        cu_seqlens = cu_seqlens.detach().cpu().numpy()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    if cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing, end at T")
    return cu


def kda_forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, lib=None):
    """Token-by-token fp64 KDA forward.

    Shapes: q, k, log_alpha [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    initial_state [N, H, dk, dv] or None (zeros).  Without ``cu_seqlens`` each
    of the B rows is one sequence (N = B).  With ``cu_seqlens`` ([N+1], int)
    B must be 1 and the T tokens are N packed sequences.

    Returns (o [B, T, H, dv], final_state [N, H, dk, dv]) as fp64 numpy arrays.
    ``lib`` selects another compiled copy of the oracle (default: the built one).
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or la.shape != q.shape:
        raise ValueError("q, k and log_alpha must share one shape")
    if v.shape[:3] != (B, T, H) or b.shape != (B, T, H):
        raise ValueError("v / beta shapes do not match q")
    cu = _seqlens(cu_seqlens, B, T)
    N = cu.shape[0] - 1
    S0 = _f64(initial_state)
    if S0 is not None and S0.shape != (N, H, dk, dv):
        raise ValueError(f"initial_state must be {(N, H, dk, dv)}, got {S0.shape}")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    S_final = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = (lib or _load()).oracle_kda_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        N, H, dk, dv, _ptr(o), _ptr(S_final),
    )
    if rc != 0:
        raise RuntimeError(f"oracle_kda_forward failed with code {rc}")
    return o, S_final


def kda_decode_step(q, k, v, log_alpha, beta, state):
    """One recurrent step for B independent sequences.

    q, k, log_alpha [B, H, dk]; v [B, H, dv]; beta [B, H]; state [B, H, dk, dv].
    A decode step is the forward recurrence on B sequences of length one.
    Returns (o [B, H, dv], new_state [B, H, dk, dv]) in fp64.
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    o, S = kda_forward(q[None], k[None], v[None], la[None], b[None],
                       initial_state=state, cu_seqlens=cu)
    return o[0], S


def kda_backward(q, k, v, log_alpha, beta, d_o, initial_state=None, d_final_state=None,
                 cu_seqlens=None, lib=None):
    """Gradients of L = <d_o, o> + <d_final_state, final_state> in fp64.

    Reverse-mode derivative of the token loop of ``kda_forward`` (same shapes and
    sequence rules; ``d_o`` like o, ``d_final_state`` like the final state, None
    for zeros).  Returns a dict with ``dq, dk, dv, dlog_alpha, dbeta`` (shaped like
    their inputs) and ``dS0`` [N, H, dk, dv], as fp64 numpy arrays.
    """
    q, k, v, la, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_o))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or la.shape != q.shape:
        raise ValueError("q, k and log_alpha must share one shape")
    if v.shape[:3] != (B, T, H) or b.shape != (B, T, H) or do.shape != v.shape:
        raise ValueError("v / beta / d_o shapes do not match q")
    cu = _seqlens(cu_seqlens, B, T)
    N = cu.shape[0] - 1
    S0, dSf = _f64(initial_state), _f64(d_final_state)
    for name, x in (("initial_state", S0), ("d_final_state", dSf)):
        if x is not None and x.shape != (N, H, dk, dv):
            raise ValueError(f"{name} must be {(N, H, dk, dv)}, got {x.shape}")
    g = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
         "dlog_alpha": np.zeros_like(la), "dbeta": np.zeros_like(b),
         "dS0": np.zeros((N, H, dk, dv), dtype=np.float64)}
    rc = (lib or _load()).oracle_kda_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, H, dk, dv,
        _ptr(do), _ptr(dSf), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
        _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dS0"]),
    )
    if rc != 0:
        raise RuntimeError(f"oracle_kda_backward failed with code {rc}")
    return g
