"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The library's waits on asynchronous copies and tensor-core commits are
bounded; when one gives up, the kernel records KDA_ERR_TIMEOUT in the
workspace status, lets its own work drain and returns, so the context stays
usable.  kda_debug_drop_copy arms one call in which a copy is left out (the
wait for it can never succeed) and the waits are capped at a few thousand
microseconds; these tests check the status, that the call ends promptly, and
that the next call on the same workspace is correct again.
"""
import time

import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from test_gpu_parity import check, oracle_chunk, to_dev

pytestmark = pytest.mark.gpu

KDA_ERR_TIMEOUT = 4


def _case():
    w = I.ChunkWorkload("fail", B=1, T=256, H=2, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.05, seed=61)
    return I.chunk_inputs(w)


def _run(x, ws):
    g = to_dev(x)
    o, S = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                         workspace=ws)
    return o, S


def test_dropped_copy_reports_timeout_then_recovers(cuda_device):
    x = _case()
    B, T, H, dk = x["q"].shape
    ws = torch.empty(kda.chunk_fwd_workspace_size(B, T, H, dk, 128, B, False, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    _run(x, ws)   # warm-up (loads and configures the kernels)
    torch.cuda.synchronize()
    assert kda.workspace_status(ws) == 0

    kda.debug_drop_copy(4_000_000)   # ~2 ms at the SM clock
    t0 = time.perf_counter()
    _run(x, ws)
    status = kda.workspace_status(ws)   # synchronises
    elapsed = time.perf_counter() - t0
    assert status == KDA_ERR_TIMEOUT
    assert elapsed < 1.0, f"the failing call took {elapsed:.3f} s"

    # the hook is one-shot: the same workspace works again, with correct results
    o, S = _run(x, ws)
    torch.cuda.synchronize()
    assert kda.workspace_status(ws) == 0
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o after recovery")
    check(S, S_ref, torch.bfloat16, "final_state after recovery")


def test_disarmed_hook_changes_nothing(cuda_device):
    x = _case()
    kda.debug_drop_copy(4_000_000)
    kda.debug_drop_copy(0)
    B, T, H, dk = x["q"].shape
    ws = torch.empty(kda.chunk_fwd_workspace_size(B, T, H, dk, 128, B, False, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    o, S = _run(x, ws)
    torch.cuda.synchronize()
    assert kda.workspace_status(ws) == 0
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o")


def test_dropped_copy_after_prefetches_recovers(cuda_device):
    """The dropped copy belongs to the first CTA's third item: the abort then
    happens with earlier stages' copies consumed and the next one prefetched,
    and the drain waits on exactly those phases."""
    w = I.ChunkWorkload("fail3", B=2, T=4096, H=4, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, seed=62)   # 512 items: several per CTA on 148 SMs
    x = I.chunk_inputs(w)
    ws = torch.empty(kda.chunk_fwd_workspace_size(2, 4096, 4, 128, 128, 2, False, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    _run(x, ws)
    assert kda.workspace_status(ws) == 0
    kda.debug_drop_copy(4_000_000)
    t0 = time.perf_counter()
    _run(x, ws)
    status = kda.workspace_status(ws)
    elapsed = time.perf_counter() - t0
    assert status == KDA_ERR_TIMEOUT
    assert elapsed < 1.0, f"the failing call took {elapsed:.3f} s"
    o, S = _run(x, ws)
    torch.cuda.synchronize()
    assert kda.workspace_status(ws) == 0
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o after recovery")
    check(S, S_ref, torch.bfloat16, "final_state after recovery")


def test_check_flag_raises_device_errors(cuda_device, monkeypatch):
    """chunk_fwd(check=True) and KDA_VALIDATE=1 turn a device-side error into KDAError."""
    w = I.ChunkWorkload("chk", B=1, T=100, H=2, dk=64, dv=64, dtype=torch.bfloat16, seed=63)
    g = to_dev(I.chunk_inputs(w))
    bad = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device="cuda")
    good = torch.tensor([0, 40, 60, 100], dtype=torch.int32, device="cuda")
    args = (g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None)
    with pytest.raises(kda.KDAError) as ei:
        kda.chunk_fwd(*args, bad, check=True)
    assert ei.value.status == 6
    kda.chunk_fwd(*args, good, check=True)   # no error
    monkeypatch.setenv("KDA_VALIDATE", "1")
    with pytest.raises(kda.KDAError):
        kda.chunk_fwd(*args, bad)
    kda.chunk_fwd(*args, bad, check=False)   # explicit opt-out: no synchronisation, no raise
    torch.cuda.synchronize()
