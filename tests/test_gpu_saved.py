"""The training pair kda_chunk_fwd_save / kda_chunk_bwd_saved: the forward keeps
what the backward would recompute, and the backward starts from it.  Outputs
and gradients are held to the oracle's bar, as for kda_chunk_fwd and
kda_chunk_bwd."""
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from test_gpu_backward import GRADS, check_all, cotangents, oracle_bwd, run_bwd
from test_gpu_parity import check, oracle_chunk, to_dev

pytestmark = pytest.mark.gpu


def _train(x, d_o, dSf):
    g = to_dev(x)
    o, S, saved = kda.chunk_fwd_train(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                                      g["cu_seqlens"])
    gr = kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o.cuda(),
                       initial_state=g["initial_state"], d_final_state=None if dSf is None else dSf.cuda(),
                       cu_seqlens=g["cu_seqlens"], saved=saved)
    torch.cuda.synchronize()
    return o.cpu(), S.cpu(), {k: (None if v is None else v.cpu()) for k, v in gr.items()}


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_saved_pair_varlen(cuda_device, dtype):
    lens = (1, 64, 0, 150, 77)
    w = I.ChunkWorkload("saved", B=1, T=sum(lens), H=3, dk=128, dv=64, dtype=dtype, s0_std=0.05,
                        lengths=lens, beta_edge_frac=0.1, seed=71)
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 710)
    o, S, gr = _train(x, d_o, dSf)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, dtype, "saved forward o")
    check(S, S_ref, dtype, "saved forward final_state")
    check_all(gr, oracle_bwd(x, d_o, dSf), dtype, "saved backward")
    # the same gradients as the backward that recomputes the forward
    again = run_bwd(x, d_o, dSf)
    for n in GRADS:
        a, b = gr[n].double(), again[n].double()
        assert float((a - b).norm() / b.norm().clamp_min(1e-30)) <= 1e-3, n


def test_saved_pair_many_items(cuda_device):
    """bf16, B=2, T=64 x 150, H=4: several items per CTA in every backward kernel."""
    w = I.ChunkWorkload("savedbig", B=2, T=64 * 150, H=4, dk=128, dv=128, dtype=torch.bfloat16, s0_std=0.01,
                        seed=72)
    x = I.chunk_inputs(w)
    d_o, dSf = cotangents(x, 720)
    _, _, gr = _train(x, d_o, dSf)
    for s, h in ((0, 0), (1, 3)):
        xs = {k: x[k][s:s + 1, :, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        xs["initial_state"] = x["initial_state"][s:s + 1, h:h + 1].contiguous()
        xs["cu_seqlens"] = None
        ref = oracle_bwd(xs, d_o[s:s + 1, :, h:h + 1].contiguous(), dSf[s:s + 1, h:h + 1].contiguous())
        part = {n: (gr[n][s:s + 1, :, h:h + 1] if n != "dS0" else gr[n][s:s + 1, h:h + 1]) for n in GRADS}
        check_all(part, ref, torch.bfloat16, f"saved seq {s} head {h}")
