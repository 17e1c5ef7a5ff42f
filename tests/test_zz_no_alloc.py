"""kda_chunk_fwd_static: the chunk forward for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plugin whose host framework owns all
device memory, a loop that cannot afford the allocator's synchronisation, a
fixed memory budget).  kda_chunk_fwd_static gives them the chunk forward with
its scratch space taken from a fixed array inside the library.  These tests
call it through the C ABI and compare its results with kda_chunk_fwd's (the
entry point with a caller-owned workspace) on two calls in a row, using the
same tolerances as the other parity tests.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda

pytestmark = pytest.mark.gpu

STATIC_BYTES = 64 << 20


def _static_fn():
    lib = kda.lib()
    fn = lib.kda_chunk_fwd_static
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.restype = i
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, vp, vp]
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_static(x):
    q, k, v = x["q"], x["k"], x["v"]
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu = x["cu_seqlens"]
    N = cu.numel() - 1 if cu is not None else B
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device="cuda")
    S = torch.empty(N, H, dk, dv, dtype=torch.float32, device="cuda")
    dt = kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32
    st = _static_fn()(_p(q), _p(k), _p(v), _p(x["log_alpha"]), _p(x["beta"]), _p(x["initial_state"]),
                      _p(cu), B, T, H, dk, dv, N, dt, _p(o), _p(S),
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o, S


def _dev(x):
    return {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in x.items()}


def _rel_l2(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _max_rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def test_static_matches_workspace_entry_point_twice(cuda_device):
    cases = [
        # first call: fixed-length bf16
        I.ChunkWorkload("na1", B=2, T=300, H=4, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, seed=61),
        # second call, different sizes: packed sequences in fp32 (the array keeps the first
        # call's contents; nothing of it may leak into this result)
        I.ChunkWorkload("na2", B=1, T=5 + 130 + 64 + 1, H=3, dk=64, dv=128, dtype=torch.float32,
                        s0_std=0.05, lengths=(5, 130, 64, 1), beta_edge_frac=0.1, seed=62),
    ]
    for w in cases:
        x = _dev(I.chunk_inputs(w))
        st, o_s, S_s = _call_static(x)
        assert st == 0, kda.lib().kda_last_error()
        o_w, S_w = kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                 x["initial_state"], x["cu_seqlens"])
        torch.cuda.synchronize()
        if w.dtype == torch.bfloat16:
            assert _rel_l2(o_s.float(), o_w.float()) <= 5e-3
            assert _rel_l2(S_s, S_w) <= 5e-3
        else:
            assert _max_rel(o_s, o_w) <= 1e-4
            assert _max_rel(S_s, S_w) <= 1e-4


def test_static_rejects_sizes_beyond_the_array(cuda_device):
    B, T, H, d = 4, 4096, 16, 128
    need = kda.chunk_fwd_workspace_size(B, T, H, d, d, B, False, torch.bfloat16)
    assert need > STATIC_BYTES
    z = torch.zeros(16, device="cuda")
    fn = _static_fn()
    p = _p(z)
    st = fn(p, p, p, p, p, None, None, B, T, H, d, d, B, kda.KDA_BF16, p, None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 5  # KDA_ERR_WORKSPACE, nothing launched
    assert b"static workspace" in kda.lib().kda_last_error()
