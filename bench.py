#!/usr/bin/env python
"""Throughput of the B200 KDA recurrence: chunkwise forward and decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  ``value`` is the chunkwise forward's throughput in
tokens/s (a token spans all H heads) summed over all ranks, on the training
shape B=4, T=4096, H=16, d_k=d_v=128, bf16 q/k/v, fp32 log_alpha/beta/state,
with its inputs resident in HBM; each rank runs its own batch (weak scaling,
no data-path collective: sequences and heads are independent).  Timing is on
the device with CUDA events on the launching stream, bracketed by a barrier
and a synchronize, max over ranks.  The line also carries:

* ``roofline``      -- the dominant kernel, timed live with events that the
                       library records between its launches (HBM-bound);
* ``path_roofline`` -- the whole forward against the algorithmic minimum
                       traffic of the method (inputs + outputs + state);
* ``decode``        -- one recurrent step for B=256, H=32, d=128 (state 512 MiB),
                       tokens/s and its HBM roofline;
* ``e2e``           -- the same forward through the public API from pinned
                       host buffers, copies in and out inside the timed region;
* ``cpu_baseline``  -- the fp64 CPU oracle on a bounded sample (rank 0, N=1);
* ``clocks``        -- SM clocks and throttle reasons sampled during timing.

``--impl reference`` times the fp64 CPU oracle instead (the reference arm), on
rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KDA tokens/s (chunk fwd & decode) at 1 B200; % bf16 TC peak / % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FLOPs per token and head of the chunk forward at MMA tile granularity
# (d_k = d_v = d, chunk C = 64): 2C(3d_k + 2d_v) + 6 d_k d_v.
def chunk_flops_per_token_head(dk, dv, C=64):
    return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ setup --
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str):
    """DRAM bytes per launch from a committed ncu capture, if its source still matches."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(kernel)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if sha != ent.get("source_sha"):
        return None
    return ent.get("bytes_per_launch_full")


class ClockSampler:
    """nvidia-smi clocks/throttle sampling in the background."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"kda_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        allrows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10:
                allrows.append(parts)
        rows = [r for r in allrows if self.uuid and self.uuid in r[1]] or allrows
        os.unlink(self.path)
        if not rows:
            return {"samples": 0}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        loaded = [x for x in sm if x > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------- our arm --
def bench_chunk(args, dev, world, rank):
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.workload)
    if w.lengths is not None:
        raise SystemExit("bench workload must be fixed-length")
    wr = I.ChunkWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank})  # own batch per rank
    x = I.chunk_inputs(wr)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    o = torch.empty(B, T, H, dv, dtype=w.dtype, device=dev)
    S = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    ws = torch.empty(kda.chunk_fwd_workspace_size(B, T, H, dk, dv, B, False, w.dtype),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                      None, o=o, final_state=S, workspace=ws)

    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for evs in stage_ev:
        for e in evs:
            e.record()  # creates the event handles
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = kda.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(args.steps):
        kda.set_stage_events(stage_ev[i])
        step()
    end.record()
    kda.set_stage_events(None)
    torch.cuda.synchronize()
    barrier(world)
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world, dev)
    stages = {name: statistics.mean(e[a].elapsed_time(e[b]) for e in stage_ev)
              for name, a, b in (("chunk_prep", 0, 1), ("intra_chunk", 1, 2), ("inter_chunk", 2, 3))}
    return dict(w=w, ms=ms, stages=stages, tokens=w.tokens, launches=3 * args.steps,
                x=x, o=o, S=S, ws=ws)


def chunk_bwd_tc_bytes_per_chunk_head(dk, dv, C=64):
    """Algorithmic bytes of the backward's three tensor-core product kernels per
    (chunk, head).  Value side: reads S, dS' (fp32 dk x dv), dU (fp32 C x dv), d_o
    (bf16 C x dv), the fp16 W, Q~, U0 tiles; writes dQ~, dW, dK^ (fp32 C x dk), dP
    (fp32 C x C), dgamma.  T-chain: reads the fp16 T, K~, V tiles, dU, dW, beta;
    writes dv (bf16), dK~ (fp32 C x dk), dA (fp32 C x C), dbeta parts.  Split
    factors: reads q, k (bf16), log_alpha, beta, dA, dP, M (fp32 C x C), dQ~, dK^,
    dK~, dgamma, dbeta parts; writes dq, dk (bf16), dlog_alpha (fp32), dbeta."""
    vside = 2 * 4 * dk * dv + 4 * C * dv + 2 * C * dv + 2 * (2 * C * dk + C * dv) + 4 * (3 * C * dk + C * C + dk)
    tchain = 2 * (C * C + C * dk + C * dv) + 4 * C * dv + 4 * C * dk + 4 * C + 2 * C * dv + 4 * (C * dk + C * C + C)
    split = (2 * 2 * C * dk + 4 * C * dk + 4 * C + 4 * 3 * C * C + 4 * (3 * C * dk + dk + C)
             + 2 * 2 * C * dk + 4 * C * dk + 4 * C)
    return vside + tchain + split


def bench_backward(args, dev, world, rank):
    """kda_chunk_bwd on the forward's workload, a seeded d_o and d_final_state."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.workload)
    wr = I.ChunkWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    x = I.chunk_inputs(wr)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gen = torch.Generator().manual_seed(5000 + rank)
    d_o = torch.randn(w.B, w.T, w.H, w.dv, generator=gen).to(w.dtype).to(dev)
    dSf = torch.randn(w.B, w.H, w.dk, w.dv, generator=gen).to(dev)
    ws = torch.empty(kda.chunk_bwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.B, False, w.dtype),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o, g["initial_state"], dSf,
                      workspace=ws)

    steps = args.bwd_steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    for evs in ev:
        for e in evs:
            e.record()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.workspace_status(ws) != 0:
        raise RuntimeError("device status set after the backward warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        kda.set_stage_events(ev[i])
        step()
    end.record()
    kda.set_stage_events(None)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / steps
    names = ("chunk_prep", "fwd_intra_chunk", "fwd_inter_chunk", "bwd_inter_chunk", "bwd_tc_products",
             "bwd_intra_chunk")
    stages = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev) for i, n in enumerate(names)}
    return dict(w=w, ms_per_step=ms, stages=stages, launches=(7 if w.dtype == torch.bfloat16 else 5) * steps)


def bench_train(args, dev, world, rank):
    """One training step on the forward's workload: kda_chunk_fwd_save, then
    kda_chunk_bwd_saved on what it kept (no forward recomputation)."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.workload)
    wr = I.ChunkWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    x = I.chunk_inputs(wr)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gen = torch.Generator().manual_seed(6000 + rank)
    d_o = torch.randn(w.B, w.T, w.H, w.dv, generator=gen).to(w.dtype).to(dev)
    dSf = torch.randn(w.B, w.H, w.dk, w.dv, generator=gen).to(dev)

    def step():
        _, _, saved = kda.chunk_fwd_train(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"])
        kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o, g["initial_state"], dSf,
                      saved=saved)
        return saved

    for _ in range(args.warmup):
        saved = step()
    torch.cuda.synchronize()
    if kda.workspace_status(saved) != 0:
        raise RuntimeError("device status set after the training-step warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for _ in range(args.bwd_steps):
        step()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / args.bwd_steps
    return dict(w=w, ms_per_step=ms)


def bench_decode(args, dev, world, rank):
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.decode_workload)
    P = 8
    d = I.decode_inputs(I.DecodeWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank}), pool=P)
    g = {k: v.to(dev) for k, v in d.items()}
    st = g["state0"].clone()
    o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)
    steps = args.decode_steps
    for i in range(args.warmup):
        j = i % P
        kda.recurrent_step(g["q"][j], g["k"][j], g["v"][j], g["log_alpha"][j], g["beta"][j], st, o=o)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        j = i % P
        kda.recurrent_step(g["q"][j], g["k"][j], g["v"][j], g["log_alpha"][j], g["beta"][j], st, o=o)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / steps
    return dict(w=w, ms_per_step=ms, launches=steps)


def bench_e2e(args, dev, world, res):
    """The forward through the public API from pinned host buffers."""
    from gated_delta_rule_108_b200 import kda

    x = res["x"]
    names = ("q", "k", "v", "log_alpha", "beta", "initial_state")
    host = {n: x[n].pin_memory() for n in names}
    devb = {n: torch.empty_like(host[n], device=dev) for n in names}
    o, S, ws = res["o"], res["S"], res["ws"]
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    S_h = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

    def step():
        for n in names:
            devb[n].copy_(host[n], non_blocking=True)
        kda.chunk_fwd(devb["q"], devb["k"], devb["v"], devb["log_alpha"], devb["beta"],
                      devb["initial_state"], None, o=o, final_state=S, workspace=ws)
        o_h.copy_(o, non_blocking=True)
        S_h.copy_(S, non_blocking=True)

    steps = max(3, min(args.steps, 10))
    for _ in range(min(args.warmup, 3)):
        step()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps):
        step()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / steps
    return ms, h2d, d2h


def cpu_oracle_rate(w, x, seqs, tokens, min_seconds=0.0):
    """Time the fp64 oracle on sequences ``seqs`` x first ``tokens`` tokens x all heads, in whole
    passes repeated until ``min_seconds`` have gone by (at least one pass).  Returns
    (tokens/s, seconds, passes, threads used)."""
    from oracle import oracle as orc
    sl = {n: x[n][seqs, :tokens] for n in ("q", "k", "v", "log_alpha", "beta")}
    S0 = None if x["initial_state"] is None else x["initial_state"][seqs]
    n_seq = len(range(*seqs.indices(w.B)))
    passes = 0
    t0 = time.perf_counter()
    while True:
        orc.kda_forward(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], S0)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    return passes * n_seq * tokens / dt, dt, passes, min(orc.num_threads(), n_seq * w.H)


def run_ours(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from gated_delta_rule_108_b200 import build
    if rank == 0:
        build.build()
    barrier(world)

    peaks, peak_kind = load_peaks()
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", ""))
    clocks = ClockSampler(uuid)
    clocks.start()
    res = bench_chunk(args, dev, world, rank)
    dec = None if args.no_decode else bench_decode(args, dev, world, rank)
    bwd = None if args.no_bwd else bench_backward(args, dev, world, rank)
    train = None if (args.no_bwd or args.no_train) else bench_train(args, dev, world, rank)
    clk = clocks.stop()
    e2e = None if args.no_e2e else bench_e2e(args, dev, world, res)

    w = res["w"]
    ms_step = res["ms"] / args.steps
    tokens_per_s = res["tokens"] * world / (ms_step / 1e3)
    th = w.tokens * w.H  # token-heads per rank per step
    eb = 2 if w.dtype == torch.bfloat16 else 4
    # algorithmic bytes (per token-head unless noted)
    in_bytes = 2 * w.dk * eb + w.dv * eb + 4 * w.dk + 4          # q, k, v, log_alpha, beta
    out_bytes = w.dv * eb                                          # o
    state_bytes = 2 * w.num_seqs * w.H * w.dk * w.dv * 4           # S0 read + final write
    n_chunks = w.num_seqs * ((w.T + 63) // 64) * w.H
    # chunk intermediates written by the intra-chunk kernel and read by the
    # inter-chunk kernel, per chunk and head: W, Q~, K^ [64 x dk], P [64 x 64],
    # U0 [64 x dv] (fp16 on the bf16 tensor-core path, fp32 on the fp32 path)
    # and gC [dk] fp32
    rec_eb = 2 if w.dtype == torch.bfloat16 else 4
    rec_bytes = rec_eb * 64 * (3 * w.dk + w.dv + 64) + 4 * w.dk
    kernels = {
        "intra_chunk": (th * in_bytes + n_chunks * rec_bytes, res["stages"]["intra_chunk"]),
        "inter_chunk": (n_chunks * rec_bytes + th * out_bytes + state_bytes, res["stages"]["inter_chunk"]),
    }
    dom = max(kernels, key=lambda k: kernels[k][1])
    dom_bytes, dom_ms = kernels[dom]
    hbm = float(peaks["hbm_gbs"])
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    path_bytes = th * (in_bytes + out_bytes) + state_bytes
    path_gbs = path_bytes / (ms_step / 1e3) / 1e9
    flops = chunk_flops_per_token_head(w.dk, w.dv) * th
    tflops = flops / (ms_step / 1e3) / 1e12
    line = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; q,k unit-norm N(0,1), v N(0,1), beta sigmoid(N(0,1)), "
                "log_alpha -exp(N(0,1))/16, S0 N(0,0.01^2))",
        "config": {
            "workload": f"{w.name}: KDA chunk fwd, B={w.B}, T={w.T}, H={w.H}, d_k=d_v={w.dk}, chunk 64, "
                        "bf16 q/k/v, fp32 log_alpha/beta/state",
            "global_batch": w.B * world, "seq_len": w.T, "heads": w.H,
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
            "l2": f"inputs larger than L2 ({th * in_bytes / 1e6:.0f} MB read per step)",
        },
        "roofline": {
            "kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic_for(dom), "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_launch": dom_bytes, "ms_per_launch": dom_ms,
        },
        "path_roofline": {
            "bound": "hbm", "achieved": path_gbs, "peak": hbm, "unit": "GB/s", "frac": path_gbs / hbm,
            "algorithmic_bytes_per_step": path_bytes,
            "tc_tflops_flop_counted": tflops,
            "tc_frac_of_bf16_peak": tflops / float(peaks["bf16_tflops"]),
        },
        "kernels_ms": res["stages"],
        "gpu_launches": res["launches"],
    }
    if dec is not None:
        dw = dec["w"]
        dbytes = dw.B * dw.H * (2 * dw.dk * dw.dv * 4 + (2 * dw.dk + 2 * dw.dv) * 2 + 4 * dw.dk + 4)
        dgbs = dbytes / (dec["ms_per_step"] / 1e3) / 1e9
        line["decode"] = {
            "workload": f"{dw.name}: kda_recurrent_step, B={dw.B}, H={dw.H}, d_k=d_v={dw.dk}, "
                        "bf16 q/k/v, fp32 state in place",
            "value": dw.B * world / (dec["ms_per_step"] / 1e3), "unit": "tokens/s",
            "ms_per_step": dec["ms_per_step"], "steps": args.decode_steps,
            "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": dgbs, "peak": hbm,
                         "unit": "GB/s", "frac": dgbs / hbm, "traffic": traffic_for("decode_step"),
                         "algorithmic_bytes_per_launch": dbytes},
        }
    if bwd is not None:
        bw = bwd["w"]
        n_ch = bw.num_seqs * ((bw.T + 63) // 64) * bw.H
        vbytes = chunk_bwd_tc_bytes_per_chunk_head(bw.dk, bw.dv) * n_ch
        vms = bwd["stages"]["bwd_tc_products"]
        vgbs = vbytes / (vms / 1e3) / 1e9
        line["chunk_bwd"] = {
            "workload": f"{bw.name}: kda_chunk_bwd (dq, dk, dv, dlog_alpha, dbeta, dS0), B={bw.B}, T={bw.T}, "
                        f"H={bw.H}, d_k=d_v={bw.dk}, bf16 q/k/v/d_o; tensor-core products (fp16 / tf32 operands, "
                        "fp32 accumulation), strong-decay chunks on CUDA cores in fp32",
            "value": bw.tokens * world / (bwd["ms_per_step"] / 1e3), "unit": "tokens/s",
            "ms_per_step": bwd["ms_per_step"], "steps": args.bwd_steps, "kernels_ms": bwd["stages"],
            "gpu_launches": bwd["launches"],
            "roofline": {"kernel": "bwd_vside_tc + bwd_tchain_tc + bwd_split_tc (the dominant stage)",
                         "bound": "hbm", "achieved": vgbs, "peak": hbm, "unit": "GB/s", "frac": vgbs / hbm,
                         "traffic": traffic_for("bwd_tc_products"), "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": vbytes, "ms_per_launch": vms},
            "strong_decay_chunks_ms": bwd["stages"]["bwd_intra_chunk"],
        }
    if train is not None:
        tw = train["w"]
        line["train_step"] = {
            "workload": f"{tw.name}: kda_chunk_fwd_save then kda_chunk_bwd_saved (forward kept for the "
                        f"backward), B={tw.B}, T={tw.T}, H={tw.H}, d_k=d_v={tw.dk}, bf16 q/k/v/d_o",
            "value": tw.tokens * world / (train["ms_per_step"] / 1e3), "unit": "tokens/s",
            "ms_per_step": train["ms_per_step"], "steps": args.bwd_steps,
        }
    if e2e is not None:
        ms_e, h2d, d2h = e2e
        line["e2e"] = {"value": res["tokens"] * world / (ms_e / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e}
    if clk is not None:
        line["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, passes, cores = cpu_oracle_rate(w, res["x"], slice(0, w.B), w.T, min_seconds=10.0)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"the whole workload ({w.B} sequences x {w.H} heads x {w.T} tokens), "
                                          f"{passes} passes in {dt:.1f} s, fp64 C oracle, OpenMP over "
                                          "(sequence, head)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------- reference arm --
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from gated_delta_rule_108_b200 import inputs as I
    from oracle import oracle as orc
    orc.build_oracle()
    w = I.workload(args.workload)
    x = I.chunk_inputs(w)
    tokens = args.reference_tokens
    for _ in range(args.warmup):
        cpu_oracle_rate(w, x, slice(0, 1), tokens)
    times = []
    cores = 1
    for _ in range(args.steps):
        _, dt, _, cores = cpu_oracle_rate(w, x, slice(0, 1), tokens)
        times.append(dt)
    ms = 1e3 * statistics.mean(times)
    value = tokens / (ms / 1e3)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": f"{w.name}: KDA chunk fwd, B={w.B}, T={w.T}, H={w.H}, d_k=d_v={w.dk}; "
                               f"each step = sequence 0, all heads, first {tokens} tokens",
                   "global_batch": w.B, "seq_len": w.T, "heads": w.H},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"sequence 0 of {w.B}, {w.H} heads, {tokens} tokens per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="C1")
    ap.add_argument("--decode-workload", default="C3")
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--reference-tokens", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward (kda_chunk_bwd) measurement")
    ap.add_argument("--bwd-steps", type=int, default=10)
    ap.add_argument("--no-train", action="store_true", help="skip the training-step (saved forward) measurement")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        log("note: fewer than 3 warm-up steps")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
