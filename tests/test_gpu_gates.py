"""Gated DeltaNet (one decay per head) and DeltaNet (no decay) through the same
kernels, against the fp64 oracle fed the gate broadcast to every key channel.

The two are the KDA recurrence with log_alpha constant across channels
(news.bugfactory.tech/news/3610, Gated DeltaNet and DeltaNet paragraphs); the
oracle pins these reductions on the CPU (tests/pins.py).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from oracle import oracle as orc
from test_gpu_parity import check, run_chunk, oracle_chunk

pytestmark = pytest.mark.gpu


def head_gate(shape, seed, div=16.0):
    g = torch.Generator().manual_seed(seed)
    return -torch.exp(torch.randn(*shape, generator=g)) / div


def with_gate(x, gate, seed):
    """Replace x's log_alpha by a per-head gate (or none); return the gate tensor
    the kernels take and the per-channel expansion the oracle takes."""
    B, T, H, dk = x["q"].shape
    if gate == "none":
        return None, torch.zeros(B, T, H, dk)
    la = head_gate((B, T, H), seed)
    return la, la[..., None].expand(B, T, H, dk).contiguous()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("gate", ["head", "none"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)], ids=["dk128dv128", "dk64dv128"])
def test_chunk_gates(cuda_device, dtype, gate, dk, dv):
    w = I.ChunkWorkload("gate", B=2, T=209, H=3, dk=dk, dv=dv, dtype=dtype, s0_std=0.05, seed=41)
    x = I.chunk_inputs(w)
    la_kernel, la_oracle = with_gate(x, gate, 411)
    xk = dict(x, log_alpha=la_kernel)
    o, S = run_chunk(xk)
    o_ref, S_ref = oracle_chunk(dict(x, log_alpha=la_oracle))
    check(o, o_ref, dtype, f"{gate} o")
    check(S, S_ref, dtype, f"{gate} final_state")


def test_chunk_head_gate_varlen(cuda_device):
    lens = (1, 64, 0, 150, 77)
    w = I.ChunkWorkload("gvl", B=1, T=sum(lens), H=2, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, lengths=lens, beta_edge_frac=0.1, seed=42)
    x = I.chunk_inputs(w)
    la_kernel, la_oracle = with_gate(x, "head", 421)
    o, S = run_chunk(dict(x, log_alpha=la_kernel))
    o_ref, S_ref = oracle_chunk(dict(x, log_alpha=la_oracle))
    check(o, o_ref, torch.bfloat16, "varlen head-gate o")
    check(S, S_ref, torch.bfloat16, "varlen head-gate final_state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("gate", ["head", "none"])
def test_decode_gates(cuda_device, dtype, gate):
    w = I.DecodeWorkload("gdec", B=5, H=3, dk=128, dv=64, steps=6, dtype=dtype, s0_std=0.1)
    d = I.decode_inputs(w, pool=6)
    st = d["state0"].cuda().clone()
    S_ref = d["state0"].double().numpy()
    for n in range(6):
        if gate == "none":
            la_k, la_o = None, torch.zeros(5, 3, 128)
        else:
            la_k = head_gate((5, 3), 430 + n)
            la_o = la_k[..., None].expand(5, 3, 128).contiguous()
        o = kda.recurrent_step(d["q"][n].cuda(), d["k"][n].cuda(), d["v"][n].cuda(),
                               None if la_k is None else la_k.cuda(), d["beta"][n].cuda(), st)
        torch.cuda.synchronize()
        o_ref, S_ref = orc.kda_decode_step(d["q"][n], d["k"][n], d["v"][n], la_o, d["beta"][n], S_ref)
        check(o, o_ref, dtype, f"{gate} decode o step {n}")
    check(st, S_ref, dtype, f"{gate} decode state")


def test_head_gate_c1_shape_sampled(cuda_device):
    """C1 sizes (B=4, T=4096, H=16, d=128, bf16) with a per-head gate."""
    w = I.workload("C1")
    x = I.chunk_inputs(w)
    la_kernel, _ = with_gate(x, "head", 441)
    o, S = run_chunk(dict(x, log_alpha=la_kernel))
    o, S = o.cpu(), S.cpu()
    for (b, h) in [(0, 0), (3, 15)]:
        xs = {kk: x[kk][b:b + 1, :, h:h + 1] for kk in ("q", "k", "v", "beta")}
        la_o = la_kernel[b:b + 1, :, h:h + 1, None].expand(1, w.T, 1, w.dk)
        o_ref, S_ref = orc.kda_forward(xs["q"], xs["k"], xs["v"], la_o, xs["beta"],
                                       x["initial_state"][b:b + 1, h:h + 1])
        check(o[b:b + 1, :, h:h + 1], o_ref, torch.bfloat16, f"head-gate C1 o ({b},{h})")
        check(S[b:b + 1, h:h + 1], S_ref, torch.bfloat16, f"head-gate C1 state ({b},{h})")
