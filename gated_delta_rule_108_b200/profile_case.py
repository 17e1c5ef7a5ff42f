"""Run one small, fixed case of a kernel of the library (for profilers).

    python -m gated_delta_rule_108_b200.profile_case decode --B 96 --H 32 --launches 3
    python -m gated_delta_rule_108_b200.profile_case chunk --B 1 --T 8192 --H 16 --launches 3
    KDA_CHUNK_PATH=fused python -m gated_delta_rule_108_b200.profile_case chunk --lengths 4096,2048 --H 32
    python -m gated_delta_rule_108_b200.profile_case chunk_bwd --B 4 --T 4096 --H 16 --launches 2

Inputs are seeded synthetic data (gated_delta_rule_108_b200.inputs); each
launch is one library call; the process synchronises and exits 0 on success.
"""
from __future__ import annotations

import argparse

import torch

from . import inputs as I
from . import kda


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["decode", "chunk", "chunk_bwd"])
    ap.add_argument("--B", type=int, default=96)
    ap.add_argument("--T", type=int, default=8192)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--dtype", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--lengths", type=str, default="",
                    help="chunk forms: comma-separated packed sequence lengths (B=1, cu_seqlens) instead of B x T")
    a = ap.parse_args()
    dt = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    if a.what == "decode":
        w = I.DecodeWorkload("profile", B=a.B, H=a.H, dk=a.d, dv=a.d, steps=a.launches, dtype=dt)
        x = {k: v.cuda() for k, v in I.decode_inputs(w, pool=1).items()}
        st = x["state0"].clone()
        for _ in range(a.launches):
            kda.recurrent_step(x["q"][0], x["k"][0], x["v"][0], x["log_alpha"][0], x["beta"][0], st)
    else:
        if a.lengths:
            lens = tuple(int(n) for n in a.lengths.split(","))
            w = I.ChunkWorkload("profile", B=1, T=sum(lens), H=a.H, dk=a.d, dv=a.d, dtype=dt, s0_std=0.01,
                                lengths=lens, seed=7)
        else:
            w = I.ChunkWorkload("profile", B=a.B, T=a.T, H=a.H, dk=a.d, dv=a.d, dtype=dt, s0_std=0.01, seed=7)
        x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in I.chunk_inputs(w).items()}
        if a.what == "chunk":
            for _ in range(a.launches):
                kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"],
                              x["cu_seqlens"])
        else:
            g = torch.Generator().manual_seed(8)
            d_o = torch.randn(x["v"].shape, generator=g).to(dt).cuda()
            for _ in range(a.launches):
                kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o, x["initial_state"])
    torch.cuda.synchronize()
    print(f"{a.what}: {a.launches} launches ok")


if __name__ == "__main__":
    main()
