"""The two calls of the boundary as declared -- kda_chunk_fwd and
kda_recurrent_step, not their gate-shaped variants that the Python binding
uses -- called through ctypes with raw device pointers and checked against the
fp64 oracle (same bars as tests/test_gpu_parity.py)."""
import ctypes

import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from oracle import oracle as orc
from test_gpu_parity import check

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("varlen", [False, True], ids=["fixed", "varlen"])
def test_kda_chunk_fwd_symbol(cuda_device, dtype, varlen):
    if varlen:
        lens = (70, 0, 129, 64)
        w = I.ChunkWorkload("abi", B=1, T=sum(lens), H=3, dk=128, dv=64, dtype=dtype, s0_std=0.05,
                            lengths=lens, seed=71)
    else:
        w = I.ChunkWorkload("abi", B=2, T=150, H=3, dk=64, dv=128, dtype=dtype, s0_std=0.05, seed=72)
    x = I.chunk_inputs(w)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    N = w.num_seqs
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=dtype, device="cuda")
    S = torch.empty(N, w.H, w.dk, w.dv, dtype=torch.float32, device="cuda")
    lib = kda.lib()
    code = kda.KDA_BF16 if dtype == torch.bfloat16 else kda.KDA_F32
    nbytes = lib.kda_chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, N, int(varlen), code)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = lib.kda_chunk_fwd(_p(g["q"]), _p(g["k"]), _p(g["v"]), _p(g["log_alpha"]), _p(g["beta"]),
                           _p(g["initial_state"]), _p(g["cu_seqlens"]), w.B, w.T, w.H, w.dk, w.dv, N,
                           code, _p(o), _p(S), _p(ws), nbytes,
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kda.KDA_OK, lib.kda_last_error()
    assert lib.kda_workspace_status(_p(ws), nbytes,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == kda.KDA_OK
    o_ref, S_ref = orc.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                   x["initial_state"], x["cu_seqlens"])
    check(o, o_ref, dtype, "o")
    check(S, S_ref, dtype, "final_state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_kda_recurrent_step_symbol(cuda_device, dtype):
    w = I.DecodeWorkload("abi", B=7, H=4, dk=128, dv=128, steps=3, dtype=dtype, s0_std=0.1, seed=73)
    d = I.decode_inputs(w, pool=3)
    st = d["state0"].cuda().clone()
    S_ref = d["state0"].double().numpy()
    lib = kda.lib()
    code = kda.KDA_BF16 if dtype == torch.bfloat16 else kda.KDA_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for n in range(3):
        q, k, v = d["q"][n].cuda(), d["k"][n].cuda(), d["v"][n].cuda()
        la, b = d["log_alpha"][n].cuda(), d["beta"][n].cuda()
        o = torch.empty(w.B, w.H, w.dv, dtype=dtype, device="cuda")
        rc = lib.kda_recurrent_step(_p(q), _p(k), _p(v), _p(la), _p(b), _p(st), w.B, w.H, w.dk, w.dv,
                                    code, _p(o), stream)
        assert rc == kda.KDA_OK, lib.kda_last_error()
        torch.cuda.synchronize()
        o_ref, S_ref = orc.kda_decode_step(d["q"][n], d["k"][n], d["v"][n], d["log_alpha"][n],
                                           d["beta"][n], S_ref)
        check(o, o_ref, dtype, f"o step {n}")
    check(st, S_ref, dtype, "state after 3 steps")
