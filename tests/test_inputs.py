"""The seeded generators: determinism, shapes and the prescribed distributions."""
import torch

from gated_delta_rule_108_b200 import inputs as I


def small(**kw):
    base = dict(name="t", B=2, T=70, H=3, dk=16, dv=8, dtype=torch.bfloat16,
                s0_std=0.01, seed=5)
    base.update(kw)
    return I.ChunkWorkload(**base)


def test_deterministic():
    a = I.chunk_inputs(small())
    b = I.chunk_inputs(small())
    for key in ("q", "k", "v", "log_alpha", "beta", "initial_state"):
        assert torch.equal(a[key], b[key]), key
    c = I.chunk_inputs(small(seed=6))
    assert not torch.equal(a["q"], c["q"])


def test_shapes_and_ranges():
    w = small()
    x = I.chunk_inputs(w)
    assert x["q"].shape == (2, 70, 3, 16) and x["q"].dtype == torch.bfloat16
    assert x["v"].shape == (2, 70, 3, 8)
    assert x["log_alpha"].dtype == torch.float32 and bool((x["log_alpha"] < 0).all())
    assert bool(((x["beta"] > 0) & (x["beta"] < 1)).all())
    assert x["initial_state"].shape == (2, 3, 16, 8)
    n = x["k"].float().norm(dim=-1)
    assert float((n - 1).abs().max()) < 1e-2  # unit norm up to bf16 rounding
    assert x["cu_seqlens"] is None


def test_varlen_and_beta_edges():
    lens = (5, 64, 0, 130)
    w = small(B=1, T=sum(lens), lengths=lens, beta_edge_frac=0.1)
    x = I.chunk_inputs(w)
    assert x["cu_seqlens"].tolist() == [0, 5, 69, 69, 199]
    per_tok = x["beta"][0]  # [T, H]
    ones = (per_tok == 1.0).all(dim=1)
    zeros = (per_tok == 0.0).all(dim=1)
    assert int(ones.sum()) == round(0.1 * w.T) and int(zeros.sum()) == round(0.1 * w.T)
    assert not bool((ones & zeros).any())


def test_named_workloads():
    c4 = I.workload("C4")
    assert len(c4.lengths) == 16 and all(1024 <= n <= 16384 for n in c4.lengths)
    assert c4.T == sum(c4.lengths)
    assert I.workload("C1").tokens == 4 * 4096
    c3 = I.workload("C3")
    assert (c3.B, c3.H, c3.dk, c3.steps) == (256, 32, 128, 1024)


def test_decode_pool():
    w = I.DecodeWorkload("d", B=3, H=2, dk=16, dv=8, steps=10)
    x = I.decode_inputs(w, pool=4)
    assert x["q"].shape == (4, 3, 2, 16) and x["state0"].shape == (3, 2, 16, 8)
    y = I.decode_inputs(w, pool=4)
    assert torch.equal(x["k"], y["k"])
