"""Thin ctypes binding of libkda_b200.so (declared in include/kda.h).

Argument marshalling only: shapes and dtypes are read off torch tensors, output
and workspace buffers are allocated with torch on the tensors' device, and the
C entry points do all of the work on the current (or given) CUDA stream.  There
is no CPU path: if the library is missing, every call raises :class:`KDAError`.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libkda_b200.so"

KDA_OK = 0
_STATUS = {
    0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
    4: "KDA_ERR_TIMEOUT", 5: "KDA_ERR_WORKSPACE", 6: "KDA_ERR_BAD_SEQLENS", 7: "KDA_ERR_RANGE",
}
KDA_F32, KDA_BF16 = 0, 1
KDA_GATE_CHANNEL, KDA_GATE_HEAD, KDA_GATE_NONE = 0, 1, 2

_lock = threading.Lock()
_lib = None


class KDAError(RuntimeError):
    """A libkda_b200 call returned a status other than KDA_OK."""

    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{_STATUS.get(status, status)}: {message}")


def library_path() -> str:
    """Path of the in-tree CUDA library (built by ``__graft_entry__.build()``)."""
    return os.environ.get("KDA_B200_LIB", os.path.join(_HERE, _LIB_NAME))


def _declare(lib):
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fp = ctypes.POINTER(f)
    lib.kda_chunk_fwd_workspace_size.restype = sz
    lib.kda_chunk_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.kda_chunk_fwd.restype = i
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                  vp, vp, vp, sz, vp]
    lib.kda_recurrent_step.restype = i
    lib.kda_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp]
    lib.kda_chunk_fwd_gated.restype = i
    lib.kda_chunk_fwd_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                        vp, vp, vp, sz, vp]
    lib.kda_recurrent_step_gated.restype = i
    lib.kda_recurrent_step_gated.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp]
    lib.kda_chunk_bwd_workspace_size.restype = sz
    lib.kda_chunk_bwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.kda_chunk_bwd.restype = i
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                  vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_chunk_bwd_gated.restype = i
    lib.kda_chunk_bwd_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                        vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_chunk_fwd_plan.restype = i
    lib.kda_chunk_fwd_plan.argtypes = [i, i, i, i, i, i, i, i, sz]
    lib.kda_chunk_fwd_fused_workspace_size.restype = sz
    lib.kda_chunk_fwd_fused_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.kda_chunk_fwd_save.restype = i
    lib.kda_chunk_fwd_save.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                       vp, vp, vp, sz, vp]
    lib.kda_chunk_bwd_saved.restype = i
    lib.kda_chunk_bwd_saved.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                        vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_workspace_status.restype = i
    lib.kda_workspace_status.argtypes = [vp, sz, vp]
    lib.kda_set_stage_events.restype = i
    lib.kda_set_stage_events.argtypes = [ctypes.POINTER(vp), i]
    lib.kda_debug_drop_copy.restype = i
    lib.kda_debug_drop_copy.argtypes = [ctypes.c_longlong]
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_last_error.argtypes = []
    lib.kda_version.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    del fp
    return lib


def lib():
    """Load (once) and return the ctypes handle of libkda_b200.so."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise KDAError(3, f"CUDA library not found at {path}; build it with "
                                  "`python -c 'import __graft_entry__ as g; g.build()'`")
            _lib = _declare(ctypes.CDLL(path))
    return _lib


def _check(status: int):
    if status != KDA_OK:
        raise KDAError(status, lib().kda_last_error().decode(errors="replace"))


def _validate_default() -> bool:
    """``KDA_VALIDATE=1`` in the environment turns on ``check`` by default."""
    return os.environ.get("KDA_VALIDATE", "0") not in ("", "0", "false", "False")


def _check_device_status(workspace: torch.Tensor, stream) -> None:
    """Synchronise on the call's stream and raise if a kernel left an error
    (bad cu_seqlens, a bounded wait that gave up, an fp16-range overflow)."""
    _check(lib().kda_workspace_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream_ptr(stream, workspace.device)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream: Optional[torch.cuda.Stream], device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _used_on(stream: Optional[torch.cuda.Stream], device, *tensors) -> None:
    """Buffers the binding allocates come from the caching allocator on the
    current stream.  When the call runs on another stream, mark them as used
    there, so that their memory is not handed out again (after the caller, or
    this function's return, drops them) before that stream's work is done."""
    if stream is None or stream.cuda_stream == torch.cuda.current_stream(device).cuda_stream:
        return
    for t in tensors:
        if t is not None:
            t.record_stream(stream)


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _dims(t: torch.Tensor, name: str, n: int):
    if t.dim() != n:
        raise ValueError(f"{name} must have {n} dimensions, got shape {tuple(t.shape)}")


def _shape(t: Optional[torch.Tensor], name: str, shape):
    """The kernels take every size from q (and v, cu_seqlens): a tensor of any
    other shape would be read or written out of bounds, so it is refused here."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _num_seqs(B: int, cu_seqlens) -> int:
    if cu_seqlens is None:
        return B
    _dims(cu_seqlens, "cu_seqlens", 1)
    if B != 1:
        raise ValueError(f"cu_seqlens requires B == 1 (sequences packed along T), got B={B}")
    if cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must hold N + 1 >= 1 offsets")
    return cu_seqlens.numel() - 1


def chunk_fwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                             num_seqs: int, varlen: bool, dtype: torch.dtype) -> int:
    """Workspace bytes ``chunk_fwd`` needs (``kda_chunk_fwd_workspace_size``)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs,
                                                  int(bool(varlen)), code))


def chunk_fwd_plan(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int, varlen: bool,
                   dtype: torch.dtype, workspace_bytes: Optional[int] = None) -> int:
    """1 if ``chunk_fwd`` with a workspace of ``workspace_bytes`` (default: the
    full ``chunk_fwd_workspace_size``) runs the fused single pass, 0 for the
    two-kernel form, -1 if neither fits (``kda_chunk_fwd_plan``)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    if workspace_bytes is None:
        workspace_bytes = chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, varlen, dtype)
    return int(lib().kda_chunk_fwd_plan(B, T, H, dk, dv, num_seqs, int(bool(varlen)), code,
                                        int(workspace_bytes)))


def chunk_fwd_fused_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                                   num_seqs: int, varlen: bool, dtype: torch.dtype) -> int:
    """Workspace bytes of the fused single pass (``kda_chunk_fwd_fused_workspace_size``;
    0 for fp32 inputs)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_fwd_fused_workspace_size(B, T, H, dk, dv, num_seqs,
                                                        int(bool(varlen)), code))


def _gate_of(log_alpha, channel_ndim: int, shape_channel, shape_head, device=None) -> int:
    """Gate kind from log_alpha's shape: None -> no gate (DeltaNet), one value
    per head -> Gated DeltaNet, one value per key channel -> KDA."""
    if log_alpha is None:
        return KDA_GATE_NONE
    if tuple(log_alpha.shape) == tuple(shape_channel):
        gate = KDA_GATE_CHANNEL
    elif tuple(log_alpha.shape) == tuple(shape_head):
        gate = KDA_GATE_HEAD
    else:
        raise ValueError(f"log_alpha must be {tuple(shape_channel)} (per channel), {tuple(shape_head)} "
                         f"(per head) or None, got {tuple(log_alpha.shape)}")
    _need(log_alpha, "log_alpha", torch.float32, device)
    return gate


def chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
              output_final_state: bool = True, o=None, final_state=None,
              workspace=None, stream=None, check: Optional[bool] = None,
              _save: bool = False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise forward (``kda_chunk_fwd_gated``).

    q, k [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    log_alpha [B, T, H, dk] (KDA), [B, T, H] (Gated DeltaNet) or None (DeltaNet);
    initial_state [N, H, dk, dv] fp32 or None; cu_seqlens int32 [N+1] or None.
    Returns (o [B, T, H, dv], final_state [N, H, dk, dv] or None).

    Errors found by the kernels while they run (cu_seqlens rejected on the
    device, a bounded wait that gave up, a bf16-path value beyond the fp16
    range) are written to the workspace's status word and are NOT raised by
    default, since reading them needs a synchronisation.  ``check=True`` (or
    ``KDA_VALIDATE=1`` in the environment) synchronises after the call and
    raises :class:`KDAError` for them; otherwise pass a ``workspace`` and read
    it later with :func:`workspace_status`.
    """
    _dims(q, "q", 4)
    _dims(v, "v", 4)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = _num_seqs(B, cu_seqlens)
    for t, n, shape in ((k, "k", (B, T, H, dk)), (v, "v", (B, T, H, dv)), (beta, "beta", (B, T, H)),
                        (initial_state, "initial_state", (N, H, dk, dv)), (o, "o", (B, T, H, dv)),
                        (final_state, "final_state", (N, H, dk, dv))):
        _shape(t, n, shape)
    dev = q.device
    gate = _gate_of(log_alpha, 4, (B, T, H, dk), (B, T, H), dev)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    for t, n, dt in ((initial_state, "initial_state", torch.float32), (o, "o", q.dtype),
                     (final_state, "final_state", torch.float32)):
        if t is not None:
            _need(t, n, dt, dev)
    made = []
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
        made.append(o)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
        made.append(final_state)
    size_fn = chunk_bwd_workspace_size if _save else chunk_fwd_workspace_size
    ws_bytes = size_fn(B, T, H, dk, dv, N, cu_seqlens is not None, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
        made.append(workspace)
    _used_on(stream, q.device, *made)
    call = lib().kda_chunk_fwd_save if _save else lib().kda_chunk_fwd_gated
    _check(call(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
        _ptr(cu_seqlens), B, T, H, dk, dv, N, _dtype_code(q), gate, _ptr(o), _ptr(final_state),
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream, q.device)))
    if check if check is not None else _validate_default():
        _check_device_status(workspace, stream)
    if _save:
        return o, final_state, workspace
    return o, final_state


def chunk_fwd_train(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                    output_final_state: bool = True, o=None, final_state=None, stream=None,
                    check: Optional[bool] = None):
    """``chunk_fwd`` for training (``kda_chunk_fwd_save``): returns (o, final_state,
    saved), where ``saved`` is a backward-sized workspace that also holds what
    ``chunk_bwd`` would recompute.  Pass it as ``chunk_bwd(..., saved=saved)`` with
    the same inputs, unchanged, to skip the recomputation."""
    return chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, output_final_state, o,
                     final_state, None, stream, check, _save=True)


def chunk_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                             num_seqs: int, varlen: bool, dtype: torch.dtype) -> int:
    """Workspace bytes ``chunk_bwd`` needs (``kda_chunk_bwd_workspace_size``)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(lib().kda_chunk_bwd_workspace_size(B, T, H, dk, dv, num_seqs,
                                                  int(bool(varlen)), code))


def chunk_bwd(q, k, v, log_alpha, beta, d_o, initial_state=None, d_final_state=None,
              cu_seqlens=None, output_d_initial_state: bool = True, workspace=None,
              stream=None, saved=None, check: Optional[bool] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Gradients of the chunkwise forward (``kda_chunk_bwd_gated``).

    Inputs as ``chunk_fwd``: log_alpha [B, T, H, dk] (KDA), [B, T, H] (Gated
    DeltaNet) or None (DeltaNet); d_o like o; d_final_state [N, H, dk, dv] fp32
    or None.  Returns a dict with dq, dk, dv (input dtype), dlog_alpha (shaped
    like log_alpha, None without a gate), dbeta (fp32) and dS0 [N, H, dk, dv]
    (fp32, or None when ``output_d_initial_state`` is false).  With ``saved``
    (the third result of ``chunk_fwd_train`` on the same inputs) the forward is
    not recomputed (``kda_chunk_bwd_saved``); ``workspace`` must then be None.
    ``check`` as in :func:`chunk_fwd`.
    """
    _dims(q, "q", 4)
    _dims(v, "v", 4)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = _num_seqs(B, cu_seqlens)
    for t, n, shape in ((k, "k", (B, T, H, dk)), (v, "v", (B, T, H, dv)), (beta, "beta", (B, T, H)),
                        (d_o, "d_o", (B, T, H, dv)), (initial_state, "initial_state", (N, H, dk, dv)),
                        (d_final_state, "d_final_state", (N, H, dk, dv))):
        _shape(t, n, shape)
    dev = q.device
    gate = _gate_of(log_alpha, 4, (B, T, H, dk), (B, T, H), dev)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o")):
        _need(t, n, q.dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    for t, n in ((initial_state, "initial_state"), (d_final_state, "d_final_state")):
        if t is not None:
            _need(t, n, torch.float32, dev)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": None if log_alpha is None else torch.empty_like(log_alpha),
         "dbeta": torch.empty_like(beta),
         "dS0": (torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
                 if output_d_initial_state else None)}
    ws_bytes = chunk_bwd_workspace_size(B, T, H, dk, dv, N, cu_seqlens is not None, q.dtype)
    call = lib().kda_chunk_bwd_gated
    if saved is not None:
        if workspace is not None:
            raise ValueError("pass either saved or workspace, not both")
        _need(saved, "saved", torch.uint8, dev)
        if saved.numel() < ws_bytes:
            raise ValueError(f"saved holds {saved.numel()} bytes; these sizes need {ws_bytes} "
                             "(it must come from chunk_fwd_train on the same inputs)")
        workspace, call = saved, lib().kda_chunk_bwd_saved
    made = list(g.values())
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
        made.append(workspace)
    _used_on(stream, q.device, *made)
    _check(call(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
        _ptr(cu_seqlens), _ptr(d_o), _ptr(d_final_state), B, T, H, dk, dv, N, _dtype_code(q), gate,
        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]),
        _ptr(g["dS0"]), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream, q.device)))
    if check if check is not None else _validate_default():
        _check_device_status(workspace, stream)
    return g


def debug_drop_copy(wait_cycles: int) -> None:
    """Arm the one-shot failure-path test hook (``kda_debug_drop_copy``)."""
    _check(lib().kda_debug_drop_copy(int(wait_cycles)))


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device status code left in ``workspace``."""
    return int(lib().kda_workspace_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream_ptr(stream, workspace.device)))


def set_stage_events(events) -> None:
    """Record ``events`` (4 ``torch.cuda.Event``s) at the stage boundaries of
    the following ``chunk_fwd`` calls on this thread; ``None`` stops it."""
    if events is None:
        _check(lib().kda_set_stage_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().kda_set_stage_events(arr, len(events)))


def recurrent_step(q, k, v, log_alpha, beta, state, o=None, stream=None) -> torch.Tensor:
    """One decoding step (``kda_recurrent_step_gated``); ``state`` is updated in place.

    q, k [B, H, dk]; v [B, H, dv]; beta [B, H]; state [B, H, dk, dv] fp32;
    log_alpha [B, H, dk] (KDA), [B, H] (Gated DeltaNet) or None (DeltaNet).
    Returns o [B, H, dv] in q's dtype.
    """
    _dims(q, "q", 3)
    _dims(v, "v", 3)
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t, n, shape in ((k, "k", (B, H, dk)), (v, "v", (B, H, dv)), (beta, "beta", (B, H)),
                        (state, "state", (B, H, dk, dv)), (o, "o", (B, H, dv))):
        _shape(t, n, shape)
    dev = q.device
    gate = _gate_of(log_alpha, 3, (B, H, dk), (B, H), dev)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if o is not None:
        _need(o, "o", q.dtype, dev)
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
        _used_on(stream, q.device, o)
    _check(lib().kda_recurrent_step_gated(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state),
        B, H, dk, dv, _dtype_code(q), gate, _ptr(o), _stream_ptr(stream, q.device)))
    return o
