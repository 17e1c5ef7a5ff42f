"""kda_chunk_bwd against the fp64 oracle's reverse-mode backward, element by
element, through the C ABI.

Every gradient (dq, dk, dv, dlog_alpha, dbeta, dS0) is held to the forward's
bar: fp32 inputs -> max relative error ||g - r||_inf / ||r||_inf <= 1e-4; bf16
inputs -> relative L2 error <= 5e-3 (the backward computes in fp32; dq, dk, dv
are rounded to bf16 on output, which alone costs ~1e-3).  The oracle runs in
fp64 on the same (dtype-rounded) inputs and cotangents.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from oracle import oracle as orc
from test_gpu_parity import check, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def cotangents(x, seed, dsf=True):
    """Seeded d_o (input dtype) and d_final_state (fp32, or None)."""
    gen = torch.Generator().manual_seed(seed)
    B, T, H, _ = x["q"].shape
    dv = x["v"].shape[-1]
    dk = x["q"].shape[-1]
    N = B if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
    d_o = torch.randn(B, T, H, dv, generator=gen).to(x["q"].dtype)
    dSf = torch.randn(N, H, dk, dv, generator=gen) if dsf else None
    return d_o, dSf


def run_bwd(x, d_o, dSf):
    g = to_dev(x)
    out = kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o.cuda(),
                        initial_state=g["initial_state"],
                        d_final_state=None if dSf is None else dSf.cuda(),
                        cu_seqlens=g["cu_seqlens"])
    torch.cuda.synchronize()
    return {k: (None if v is None else v.cpu()) for k, v in out.items()}


def oracle_bwd(x, d_o, dSf):
    return orc.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                            initial_state=x["initial_state"], d_final_state=dSf,
                            cu_seqlens=x["cu_seqlens"])


def check_all(got, ref, dtype, tag):
    errs = {}
    for n in GRADS:
        # dlog_alpha, dbeta and dS0 are fp32 outputs for both input dtypes
        errs[n] = check(got[n], ref[n], dtype, f"{tag} {n}")
    return errs


SHAPES = [(64, 64), (64, 128), (128, 64), (128, 128)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"dk{a}dv{b}" for a, b in SHAPES])
def test_chunk_bwd_small(cuda_device, dtype, dk, dv):
    # 3 full chunks and a ragged tail of 17 tokens, 2 sequences, 3 heads
    w = I.ChunkWorkload("bwd", B=2, T=209, H=3, dk=dk, dv=dv, dtype=dtype, s0_std=0.05, seed=51)
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 510)
    check_all(run_bwd(x, d_o, dSf), oracle_bwd(x, d_o, dSf), dtype, f"{dk}x{dv}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_chunk_bwd_varlen_edges(cuda_device, dtype):
    """Packed sequences of 1, 64, 0, 150 and 77 tokens; 10% beta = 1, 10% beta = 0."""
    lens = (1, 64, 0, 150, 77)
    w = I.ChunkWorkload("bvl", B=1, T=sum(lens), H=2, dk=128, dv=128, dtype=dtype, s0_std=0.05,
                        lengths=lens, beta_edge_frac=0.1, seed=52)
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 520)
    got, ref = run_bwd(x, d_o, dSf), oracle_bwd(x, d_o, dSf)
    check_all(got, ref, dtype, "varlen")
    # the empty sequence passes its final-state cotangent straight through
    np.testing.assert_array_equal(got["dS0"][2].numpy(), dSf[2].numpy())


def test_chunk_bwd_no_state_cotangents(cuda_device):
    """No initial state, no final-state cotangent (the common training call)."""
    w = I.ChunkWorkload("bns", B=1, T=130, H=2, dk=64, dv=64, dtype=torch.float32, s0_std=0.0, seed=53)
    x = I.chunk_inputs(w)
    d_o, _ = cotangents(x, 530, dsf=False)
    check_all(run_bwd(x, d_o, None), oracle_bwd(x, d_o, None), torch.float32, "no-state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_chunk_bwd_strong_decay(cuda_device, dtype):
    """Decay strong enough that the split factors would overflow: the exact
    pairwise path (every exponent <= 0) must be taken and still agree."""
    w = I.ChunkWorkload("bsd", B=1, T=150, H=2, dk=128, dv=64, dtype=dtype, s0_std=0.05, seed=54)
    x = I.chunk_inputs(w)
    gen = torch.Generator().manual_seed(541)
    # per-token log-decay down to about -8 on a few channels: ~ -250 over 32 tokens
    la = -torch.rand(x["log_alpha"].shape, generator=gen) * 0.3
    la[..., :4] = -8.0 * torch.rand(la[..., :4].shape, generator=gen)
    x["log_alpha"] = la.contiguous()
    d_o, dSf = cotangents(x, 542)
    check_all(run_bwd(x, d_o, dSf), oracle_bwd(x, d_o, dSf), dtype, "strong")


def test_chunk_bwd_c1_sampled(cuda_device):
    """bf16, B=4, T=4096, H=16, d=128 (the prefill workload): the backward of the
    whole batch on the GPU, three (sequence, head) pairs against the oracle."""
    w = I.workload("C1")
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 550)
    got = run_bwd(x, d_o, dSf)
    for (s, h) in ((0, 0), (2, 7), (3, 15)):
        xs = {k: x[k][s:s + 1, :, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        xs["initial_state"] = x["initial_state"][s:s + 1, h:h + 1].contiguous()
        xs["cu_seqlens"] = None
        ref = oracle_bwd(xs, d_o[s:s + 1, :, h:h + 1].contiguous(), dSf[s:s + 1, h:h + 1].contiguous())
        part = {n: (got[n][s:s + 1, :, h:h + 1] if n != "dS0" else got[n][s:s + 1, h:h + 1])
                for n in GRADS}
        check_all(part, ref, torch.bfloat16, f"C1 seq {s} head {h}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("gate", ["head", "none"])
def test_chunk_bwd_gates(cuda_device, dtype, gate):
    """Gated DeltaNet (one log-decay per head) and DeltaNet (none) through the
    backward.  The oracle takes the gate broadcast to every channel; a per-head
    log-decay's cotangent is the sum of the per-channel ones (chain rule)."""
    w = I.ChunkWorkload("bgate", B=2, T=150, H=2, dk=128, dv=64, dtype=dtype, s0_std=0.05, seed=56)
    x = I.chunk_inputs(w)
    B, T, H, dk = x["q"].shape
    if gate == "head":
        gen = torch.Generator().manual_seed(561)
        la = -torch.exp(torch.randn(B, T, H, generator=gen)) / 16
        la_full = la[..., None].expand(B, T, H, dk).contiguous()
    else:
        la, la_full = None, torch.zeros(B, T, H, dk)
    d_o, dSf = cotangents(x, 562)
    got = run_bwd(dict(x, log_alpha=la), d_o, dSf)
    ref = oracle_bwd(dict(x, log_alpha=la_full), d_o, dSf)
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        check(got[n], ref[n], dtype, f"{gate} {n}")
    if gate == "head":
        assert got["dlog_alpha"].shape == (B, T, H)
        check(got["dlog_alpha"], ref["dlog_alpha"].sum(-1), dtype, "head dlog_alpha")
    else:
        assert got["dlog_alpha"] is None


def test_chunk_bwd_c4_varlen_sampled(cuda_device):
    """The packed varlen workload (16 sequences of 1,024..16,384 tokens, H=32,
    bf16, 10% beta = 1 and 10% beta = 0): the backward of the whole pack on the
    GPU; the shortest and the longest sequence, one head each, against the oracle."""
    w = I.workload("C4")
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 570)
    got = run_bwd(x, d_o, dSf)
    cu = x["cu_seqlens"].tolist()
    lens = [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]
    for s, h in ((lens.index(min(lens)), 3), (lens.index(max(lens)), 29)):
        a, b = cu[s], cu[s + 1]
        xs = {k: x[k][:, a:b, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        xs["initial_state"] = x["initial_state"][s:s + 1, h:h + 1].contiguous()
        xs["cu_seqlens"] = None
        ref = oracle_bwd(xs, d_o[:, a:b, h:h + 1].contiguous(), dSf[s:s + 1, h:h + 1].contiguous())
        part = {n: (got[n][:, a:b, h:h + 1] if n != "dS0" else got[n][s:s + 1, h:h + 1]) for n in GRADS}
        check_all(part, ref, torch.bfloat16, f"C4 seq {s} (len {b - a}) head {h}")


def test_chunk_bwd_mixed_strong_chunks_many_items(cuda_device):
    """About eight (chunk, head) items per CTA, with strong-decay chunks among the ordinary ones:
    every third chunk of head 0 and every other chunk of head 2 (B=1, T=300 chunks, H=4, bf16).
    The per-item kernels walk their items in turn, skip the flagged chunks and fetch the next
    unflagged one ahead; heads 0 and 2 go against the oracle whole."""
    nch = 300
    w = I.ChunkWorkload("bmix", B=1, T=64 * nch, H=4, dk=128, dv=64, dtype=torch.bfloat16, s0_std=0.05,
                        seed=59)
    x = I.chunk_inputs(w)
    la = x["log_alpha"].clone()
    gen = torch.Generator().manual_seed(591)
    chunk = torch.arange(w.T) // 64
    # per-token log-decay down to -8 on four channels: |g - g_m| far above the split limit
    for h, strong in ((0, chunk % 3 == 1), (2, chunk % 2 == 0)):
        la[0, strong, h, :4] = -8.0 * torch.rand(int(strong.sum()), 4, generator=gen)
    x["log_alpha"] = la.contiguous()
    d_o, dSf = cotangents(x, 592)
    got = run_bwd(x, d_o, dSf)
    for h in (0, 2):
        xs = {k: x[k][:, :, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        xs["initial_state"] = x["initial_state"][:, h:h + 1].contiguous()
        xs["cu_seqlens"] = None
        ref = oracle_bwd(xs, d_o[:, :, h:h + 1].contiguous(), dSf[:, h:h + 1].contiguous())
        part = {n: (got[n][:, :, h:h + 1] if n != "dS0" else got[n][:, h:h + 1]) for n in GRADS}
        check_all(part, ref, torch.bfloat16, f"mixed head {h}")
