"""The fused single-pass form of the bf16 chunk forward (kda_chunk_fwd_plan == 1:
one CTA per (sequence, head) pair, each chunk's intermediates kept on chip)
against the fp64 oracle, on the cases the two-kernel form is checked on.  It
runs when the workspace is too small for the two-kernel form's records, or
when KDA_CHUNK_PATH=fused forces it."""
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from test_gpu_parity import check, oracle_chunk, rel_l2, run_chunk, to_dev

pytestmark = pytest.mark.gpu

SHAPES = [(64, 64), (64, 128), (128, 64), (128, 128)]


@pytest.fixture
def fused(monkeypatch):
    monkeypatch.setenv("KDA_CHUNK_PATH", "fused")


@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"dk{a}dv{b}" for a, b in SHAPES])
def test_fused_small(cuda_device, fused, dk, dv):
    w = I.ChunkWorkload("small", B=2, T=209, H=3, dk=dk, dv=dv, dtype=torch.bfloat16, s0_std=0.05, seed=21)
    assert kda.chunk_fwd_plan(w.B, w.T, w.H, dk, dv, w.B, False, w.dtype) == 1   # forced
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o")
    check(S, S_ref, torch.bfloat16, "final_state")


def test_fused_varlen_edges(cuda_device, fused):
    lens = (1, 63, 64, 65, 0, 130, 200, 0)
    w = I.ChunkWorkload("vl", B=1, T=sum(lens), H=2, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, lengths=lens, beta_edge_frac=0.1, seed=24)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "varlen o")
    check(S, S_ref, torch.bfloat16, "varlen final_state")
    # empty sequences pass their state through unchanged
    assert torch.equal(S[4].cpu(), x["initial_state"][4]) and torch.equal(S[7].cpu(), x["initial_state"][7])


@pytest.mark.parametrize("gate", ["head", "none"])
def test_fused_gate_shapes(cuda_device, fused, gate):
    w = I.ChunkWorkload("g", B=2, T=150, H=2, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.05, seed=41)
    x = I.chunk_inputs(w)
    g = to_dev(x)
    la = g["log_alpha"][..., 0].contiguous() if gate == "head" else None
    o, S = kda.chunk_fwd(g["q"], g["k"], g["v"], la, g["beta"], g["initial_state"])
    torch.cuda.synchronize()
    xr = dict(x)
    xr["log_alpha"] = (x["log_alpha"][..., :1].expand_as(x["log_alpha"]).contiguous() if gate == "head"
                       else torch.zeros_like(x["log_alpha"]))
    o_ref, S_ref = oracle_chunk(xr)
    check(o, o_ref, torch.bfloat16, f"{gate} o")
    check(S, S_ref, torch.bfloat16, f"{gate} final_state")


@pytest.mark.parametrize("where", ["all_channels", "few_channels"])
def test_fused_strong_decay(cuda_device, fused, where):
    w = I.ChunkWorkload("strong", B=2, T=200, H=2, dk=128, dv=64, dtype=torch.bfloat16, s0_std=0.05, seed=28)
    x = I.chunk_inputs(w)
    gen = torch.Generator().manual_seed(281)
    strong = -4.0 * torch.exp(0.2 * torch.randn(x["log_alpha"].shape, generator=gen))
    if where == "all_channels":
        x["log_alpha"] = strong
    else:
        x["log_alpha"][:, :, 1, [5, 77]] = strong[:, :, 1, [5, 77]]
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, f"{where} o")
    check(S, S_ref, torch.bfloat16, f"{where} final_state")


def test_fused_state_in_place_and_zero_state(cuda_device, fused):
    w = I.ChunkWorkload("alias", B=2, T=100, H=2, dk=64, dv=64, dtype=torch.bfloat16, s0_std=0.05, seed=26)
    x = I.chunk_inputs(w)
    o_ref, S_ref = oracle_chunk(x)
    g = to_dev(x)
    st = g["initial_state"].clone()
    kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], st, final_state=st)
    torch.cuda.synchronize()
    check(st, S_ref, torch.bfloat16, "aliased final_state")
    x0 = dict(x, initial_state=None)
    o0, S0 = run_chunk(x0)
    o_ref0, S_ref0 = oracle_chunk(x0)
    check(o0, o_ref0, torch.bfloat16, "zero-state o")
    check(S0, S_ref0, torch.bfloat16, "zero-state final_state")


def test_small_workspace_runs_the_fused_pass(cuda_device, monkeypatch):
    """With the full workspace the split form runs; with only the fused pass's
    workspace (header, chunk table, pair order) the fused pass runs by itself,
    and the two agree with each other and with the oracle."""
    monkeypatch.delenv("KDA_CHUNK_PATH", raising=False)
    lens = (150, 0, 1, 70, 129)
    w = I.ChunkWorkload("ws", B=1, T=sum(lens), H=4, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.05,
                        lengths=lens, seed=31)
    N = len(lens)
    full = kda.chunk_fwd_workspace_size(1, w.T, w.H, 128, 128, N, True, w.dtype)
    small = kda.chunk_fwd_fused_workspace_size(1, w.T, w.H, 128, 128, N, True, w.dtype)
    assert 0 < small < full
    assert kda.chunk_fwd_plan(1, w.T, w.H, 128, 128, N, True, w.dtype) == 0
    assert kda.chunk_fwd_plan(1, w.T, w.H, 128, 128, N, True, w.dtype, small) == 1
    assert kda.chunk_fwd_plan(1, w.T, w.H, 128, 128, N, True, w.dtype, small - 4) == -1
    assert kda.chunk_fwd_plan(1, w.T, w.H, 128, 128, N, True, torch.float32) == 0
    assert kda.chunk_fwd_fused_workspace_size(1, w.T, w.H, 128, 128, N, True, torch.float32) == 0
    x = I.chunk_inputs(w)
    g = to_dev(x)
    args = (g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"], g["cu_seqlens"])
    ws_small = torch.empty(small, dtype=torch.uint8, device="cuda")
    of, Sf = kda.chunk_fwd(*args, workspace=ws_small, check=True)
    os_, Ss = kda.chunk_fwd(*args, check=True)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(x)
    check(of, o_ref, torch.bfloat16, "fused o")
    check(Sf, S_ref, torch.bfloat16, "fused final_state")
    check(os_, o_ref, torch.bfloat16, "split o")
    assert rel_l2(of.float().cpu(), os_.float().cpu()) < 2e-3
    assert rel_l2(Sf.cpu(), Ss.cpu()) < 2e-3
    # a workspace below both sizes is refused on the host
    with pytest.raises(kda.KDAError) as ei:
        kda.chunk_fwd(*args, workspace=torch.empty(small - 256, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == 5


def test_fused_many_pairs_agrees_with_split(cuda_device, monkeypatch):
    w = I.ChunkWorkload("many", B=40, T=150, H=8, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.05, seed=30)
    x = I.chunk_inputs(w)
    monkeypatch.setenv("KDA_CHUNK_PATH", "fused")
    of, Sf = run_chunk(x)
    monkeypatch.setenv("KDA_CHUNK_PATH", "split")
    os_, Ss = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(of, o_ref, torch.bfloat16, "fused o")
    check(Sf, S_ref, torch.bfloat16, "fused final_state")
    assert rel_l2(of.float().cpu(), os_.float().cpu()) < 2e-3
    assert rel_l2(Sf.cpu(), Ss.cpu()) < 2e-3
