"""The precision choices of the kernels, checked in the rounding model
(precision_model.py) against the fp64 oracle on small seeded inputs."""
import numpy as np
import torch

from gated_delta_rule_108_b200 import inputs as I
from oracle import oracle as orc
import precision_model as pm


def _heads(w, nheads):
    x = I.chunk_inputs(w)
    o_ref, S_ref = orc.kda_forward(x["q"][:1], x["k"][:1], x["v"][:1], x["log_alpha"][:1], x["beta"][:1],
                                   None if x["initial_state"] is None else x["initial_state"][:1])
    f = lambda t: t.double().numpy()
    for h in range(nheads):
        S0 = f(x["initial_state"][0, h]) if x["initial_state"] is not None else np.zeros((w.dk, w.dv))
        yield ((f(x["q"][0, :, h]), f(x["k"][0, :, h]), f(x["v"][0, :, h]), f(x["log_alpha"][0, :, h]),
                f(x["beta"][0, :, h]), S0), o_ref[0, :, h])


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _max_rel(a, b):
    return float(np.abs(a - b).max() / np.abs(b).max())


def test_bf16_plan_costs_only_the_output_rounding():
    """tf32 split factors, fp16 intermediates: relative L2 of o near bf16 output rounding alone
    (about 1.7e-3), well inside the 5e-3 bar."""
    w = I.ChunkWorkload("pm1", B=1, T=256, H=2, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.01, seed=1)
    for args, o_ref in _heads(w, 2):
        o, _ = pm.bf16_path_head(*args)
        assert _rel_l2(o, o_ref) < 2.5e-3
        # bf16 everywhere would sit close to the bar
        o_b, _ = pm.bf16_path_head(*args, ops=pm.bf16, mid=pm.bf16)
        assert _rel_l2(o_b, o_ref) > 1.7 * _rel_l2(o, o_ref)


def test_product_form_inverse_breaks_where_the_blocked_form_holds():
    """Correlated keys, beta = 1, almost no decay: the product form's powers of A overflow
    (non-finite output); the blocked form with exact diagonal blocks stays at the bar."""
    q, k, v, la, beta = pm.correlated_keys(T=256)
    o_ref, _ = orc.kda_forward(*(torch.from_numpy(a)[None, :, None].float() for a in (q, k, v, la)),
                               torch.from_numpy(beta)[None, :, None].float(), None)
    o_ref = o_ref[0, :, 0]
    S0 = np.zeros((128, 128))
    with np.errstate(all="ignore"):
        o_prod, _ = pm.bf16_path_head(q, k, v, la, beta, S0, inv=pm.inv_product, inv_rnd=pm.fp16)
    assert not np.all(np.isfinite(o_prod)) or _rel_l2(o_prod, o_ref) > 1e-1
    o_blk, _ = pm.bf16_path_head(q, k, v, la, beta, S0, inv=pm.inv_blocked, inv_rnd=pm.fp16)
    o_ex, _ = pm.bf16_path_head(q, k, v, la, beta, S0)
    assert _rel_l2(o_blk, o_ref) < 5e-3
    assert _rel_l2(o_blk, o_ref) < 1.5 * _rel_l2(o_ex, o_ref)


def test_fp32_path_needs_split_tf32_products():
    """Single tf32 products miss the fp32 bar (max-relative 1e-4); split products meet it."""
    w = I.workload("C0")
    for args, o_ref in _heads(w, 2):
        o1, _ = pm.fp32_path_head(*args, mm=pm.mm_tf32)
        o3, _ = pm.fp32_path_head(*args, mm=pm.mm_split_tf32)
        assert _max_rel(o1, o_ref) > 1e-4
        assert _max_rel(o3, o_ref) < 1e-5
