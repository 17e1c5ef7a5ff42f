#!/usr/bin/env python
"""Throughput of the B200 KDA recurrence: chunkwise forward and decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  ``value`` is the chunkwise forward's throughput in
tokens/s (a token spans all H heads) summed over all ranks, on the largest
single-GPU workload: 16 packed sequences of 1,024-16,384 tokens (about 147 k
tokens), H=32, d_k=d_v=128, bf16 q/k/v, fp32 log_alpha/beta/state, with its
inputs resident in HBM.  Each rank runs its own batch (weak scaling, no
data-path collective: sequences and heads are independent).  Timing is on the
device with CUDA events on the launching stream, bracketed by a barrier and a
synchronize, max over ranks.  The line also carries:

* ``roofline``      -- the dominant kernel, timed live with events that the
                       library records between its launches, against the HBM
                       bytes the method itself moves through that kernel;
* ``path_roofline`` -- the whole forward against the algorithmic minimum
                       traffic of the method (inputs + outputs + state), and
                       FLOP-counted against the bf16 tensor-core peak;
* ``c1``, ``c2``    -- the same figures on the training shape (B=4, T=4096,
                       H=16) and on one 65,536-token sequence (H=32);
* ``c4_fused``      -- the headline workload with the fused single pass forced
                       (kda_chunk_fwd runs the two-kernel form by itself);
* ``decode``        -- 1,024 consecutive recurrent steps for B=256, H=32, d=128
                       (state 512 MiB), tokens/s and the HBM roofline;
* ``chunk_bwd``     -- the backward on the training shape;
* ``e2e``           -- the headline forward through the public API from pinned
                       host buffers, copies in and out inside the timed region;
* ``cpu_baseline``  -- the fp64 CPU oracle on a bounded sample (rank 0, N=1);
* ``clocks``        -- SM clocks and throttle reasons sampled during timing.

``--impl reference`` times the fp64 CPU oracle instead (the reference arm), on
rank 0 only.  ``--gpus N`` without a torchrun environment starts N ranks
itself under torch.distributed.run.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import socket
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
CHUNK = 64


# FLOPs per token and head of the chunk forward at MMA tile granularity
# (d_k = d_v = d, chunk C = 64): 2C(3d_k + 2d_v) + 6 d_k d_v.
def chunk_flops_per_token_head(dk, dv, C=CHUNK):
    return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ setup --
def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_under_torchrun(gpus: int) -> int:
    """Run this script as ``gpus`` ranks under torch.distributed.run (same
    arguments); returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def dist_setup(use_cuda: bool = True):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if use_cuda:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
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


def traffic_per_unit(kernel: str):
    """DRAM bytes per unit of work (a (chunk, head) item; a (sequence, head)
    pair for decode) from a committed ncu capture, if its source still matches."""
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
    return ent.get("bytes_per_unit")


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


# ---------------------------------------------------- workload arithmetic --
def seq_lengths(w):
    return list(w.lengths) if w.lengths is not None else [w.T] * w.B


def chunk_units(w) -> int:
    """(chunk, head) work items of a chunk-forward workload."""
    return sum((n + CHUNK - 1) // CHUNK for n in seq_lengths(w)) * w.H


def method_bytes(w):
    """Algorithmic HBM bytes of the chunk forward, by the kernel that moves them:
    the intra-chunk kernel reads q, k, v, log_alpha, beta; the inter-chunk
    kernel writes o and reads / writes the states.  Per token-head:
    (2 d_k + d_v) e + 4 d_k + 4 in, d_v e out (e = element bytes)."""
    eb = 2 if w.dtype == torch.bfloat16 else 4
    th = w.tokens * w.H
    reads = th * ((2 * w.dk + w.dv) * eb + 4 * w.dk + 4)
    o = th * w.dv * eb
    state = (2 if w.s0_std > 0 else 1) * w.num_seqs * w.H * w.dk * w.dv * 4
    return {"intra_chunk": reads, "inter_chunk": o + state, "total": reads + o + state}


def record_bytes_per_unit(w) -> int:
    """Chunk intermediates the intra-chunk kernel writes and the inter-chunk
    kernel reads, per (chunk, head): W, Q~, K^ [64 x dk], P [64 x 64], U0
    [64 x dv] (fp16 on the bf16 tensor-core path, fp32 on the fp32 path) and
    gamma_C [dk] fp32."""
    rec_eb = 2 if w.dtype == torch.bfloat16 else 4
    return rec_eb * CHUNK * (3 * w.dk + w.dv + CHUNK) + 4 * w.dk


def describe(w) -> str:
    dt = "bf16" if w.dtype == torch.bfloat16 else "fp32"
    if w.lengths is not None:
        shape = (f"{len(w.lengths)} packed sequences (cu_seqlens), lengths {min(w.lengths)}-{max(w.lengths)}, "
                 f"{w.tokens} tokens")
    else:
        shape = f"B={w.B}, T={w.T}"
    return (f"{w.name}: KDA chunk fwd, {shape}, H={w.H}, d_k={w.dk}, d_v={w.dv}, chunk 64, {dt} q/k/v, "
            f"fp32 log_alpha/beta/state")


def data_recipe(w) -> str:
    s = (f"synthetic (seeded; q,k unit-norm N(0,1), v N(0,1), beta sigmoid(N({w.beta_mu:g},1)), "
         f"log_alpha -exp(N(0,1))/{w.la_div:g}, S0 " + (f"N(0,{w.s0_std:g}^2)" if w.s0_std > 0 else "0"))
    if w.beta_edge_frac > 0:
        s += f"; {w.beta_edge_frac:.0%} of tokens beta=1 and a disjoint {w.beta_edge_frac:.0%} beta=0"
    return s + ")"


def rank_workload(w, rank: int):
    """Each rank draws its own batch of the same shape (weak scaling)."""
    if rank == 0:
        return w
    return dataclasses.replace(w, seed=w.seed + 1000 * rank, lengths_from=None)


# --------------------------------------------------------------- our arm --
def bench_chunk(name, steps, warmup, dev, world, rank, dtype=None):
    """Time kda_chunk_fwd on one workload (its shape in another input dtype if
    given); per-stage times from library events."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(name)
    if dtype is not None and dtype != w.dtype:
        w = dataclasses.replace(w, dtype=dtype, name=f"{w.name} ({'fp32' if dtype == torch.float32 else 'bf16'})")
    x = I.chunk_inputs(rank_workload(w, rank))
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    varlen = g["cu_seqlens"] is not None
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=w.dtype, device=dev)
    S = torch.empty(w.num_seqs, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)
    ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.num_seqs, varlen, w.dtype),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                      g["cu_seqlens"], o=o, final_state=S, workspace=ws)

    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for evs in stage_ev:
        for e in evs:
            e.record()  # creates the event handles
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    status = kda.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"{name}: device status {status} after warm-up")

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        kda.set_stage_events(stage_ev[i])
        step()
    end.record()
    kda.set_stage_events(None)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / steps
    if kda.workspace_status(ws) != 0:
        raise RuntimeError(f"{name}: device status set during timing")
    stages = {st: statistics.mean(e[a].elapsed_time(e[b]) for e in stage_ev)
              for st, a, b in (("chunk_prep", 0, 1), ("intra_chunk", 1, 2), ("inter_chunk", 2, 3))}
    return dict(w=w, ms=ms, stages=stages, launches=3 * steps, x=x, g=g, o=o, S=S, ws=ws)


def chunk_summary(res, world, peaks, peak_kind):
    """Throughput and rooflines of one timed chunk-forward workload."""
    w, ms = res["w"], res["ms"]
    units = chunk_units(w)
    mb = method_bytes(w)
    rec = record_bytes_per_unit(w) * units
    hbm = float(peaks["hbm_gbs"])
    kern = {k: res["stages"][k] for k in ("intra_chunk", "inter_chunk")}
    dom = max(kern, key=kern.get)
    dom_ms = kern[dom]
    achieved = mb[dom] / (dom_ms / 1e3) / 1e9
    tpu = traffic_per_unit(dom if w.dtype == torch.bfloat16 else dom + "_f32")
    path_gbs = mb["total"] / (ms / 1e3) / 1e9
    th = w.tokens * w.H
    tflops = chunk_flops_per_token_head(w.dk, w.dv) * th / (ms / 1e3) / 1e12
    # the binding roofline of the whole path: min(tensor peak, HBM bandwidth x arithmetic intensity)
    ai = chunk_flops_per_token_head(w.dk, w.dv) * th / mb["total"]
    bound_tflops = min(float(peaks["bf16_tflops"]), hbm * ai / 1e3)
    return {
        "workload": describe(w),
        "value": w.tokens * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "token_heads_per_step": th, "chunk_head_items": units,
        "kernels_ms": res["stages"],
        "roofline": {
            "kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": None if tpu is None else tpu * units,
            "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_launch": mb[dom], "ms_per_launch": dom_ms,
            "intermediate_bytes_per_launch": rec,
            "intermediate_note": "chunk records written by intra_chunk and read by inter_chunk "
                                 "(not method bytes; not counted in achieved)",
        },
        "path_roofline": {
            "bound": "hbm", "achieved": path_gbs, "peak": hbm, "unit": "GB/s", "frac": path_gbs / hbm,
            "algorithmic_bytes_per_step": mb["total"],
            "tc_tflops_flop_counted": tflops,
            "tc_frac_of_bf16_peak": tflops / float(peaks["bf16_tflops"]),
            "binding_roofline_tflops": bound_tflops,
            "frac_of_binding_roofline": tflops / bound_tflops,
        },
    }


def chunk_bwd_tc_bytes_per_chunk_head(dk, dv, C=CHUNK):
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


def bench_backward(args, dev, world, rank, peaks, peak_kind):
    """kda_chunk_bwd on the training shape, a seeded d_o and d_final_state."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.bwd_workload)
    x = I.chunk_inputs(rank_workload(w, rank))
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gen = torch.Generator().manual_seed(5000 + rank)
    d_o = torch.randn(w.B, w.T, w.H, w.dv, generator=gen).to(w.dtype).to(dev)
    dSf = torch.randn(w.num_seqs, w.H, w.dk, w.dv, generator=gen).to(dev)
    varlen = g["cu_seqlens"] is not None
    ws = torch.empty(kda.chunk_bwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.num_seqs, varlen, w.dtype),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o, g["initial_state"], dSf,
                      g["cu_seqlens"], workspace=ws)

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
    units = chunk_units(w)
    vbytes = chunk_bwd_tc_bytes_per_chunk_head(w.dk, w.dv) * units
    vms = stages["bwd_tc_products"]
    vgbs = vbytes / (vms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    tpu = traffic_per_unit("bwd_tc_products")
    return {
        "workload": f"{w.name}: kda_chunk_bwd (dq, dk, dv, dlog_alpha, dbeta, dS0), B={w.B}, T={w.T}, "
                    f"H={w.H}, d_k=d_v={w.dk}, bf16 q/k/v/d_o; tensor-core products (fp16 / tf32 operands, "
                    "fp32 accumulation), strong-decay chunks on CUDA cores in fp32",
        "value": w.tokens * world / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": ms, "steps": steps, "kernels_ms": stages,
        "gpu_launches": (8 if w.dtype == torch.bfloat16 else 5) * steps,
        "roofline": {"kernel": "bwd_vside_tc + bwd_tchain_tc + bwd_split_tc (the dominant stage)",
                     "bound": "hbm", "achieved": vgbs, "peak": hbm, "unit": "GB/s", "frac": vgbs / hbm,
                     "traffic": None if tpu is None else tpu * units, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": vbytes, "ms_per_launch": vms},
        "strong_decay_chunks_ms": stages["bwd_intra_chunk"],
    }


def bench_train(args, dev, world, rank):
    """One training step on the backward's workload: kda_chunk_fwd_save (the
    forward that keeps T, the tiles and the chunk-start states), then
    kda_chunk_bwd_saved on what it kept, so the backward recomputes nothing."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.bwd_workload)
    x = I.chunk_inputs(rank_workload(w, rank))
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    gen = torch.Generator().manual_seed(6000 + rank)
    d_o = torch.randn(w.B, w.T, w.H, w.dv, generator=gen).to(w.dtype).to(dev)
    dSf = torch.randn(w.num_seqs, w.H, w.dk, w.dv, generator=gen).to(dev)

    def step():
        _, _, saved = kda.chunk_fwd_train(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                          g["initial_state"], g["cu_seqlens"])
        kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o, g["initial_state"], dSf,
                      g["cu_seqlens"], saved=saved)
        return saved

    saved = None
    for _ in range(args.warmup):
        saved = step()
    torch.cuda.synchronize()
    if saved is not None and kda.workspace_status(saved) != 0:
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
    launches = 3 + (5 if w.dtype == torch.bfloat16 else 2)   # prep, K1, K2; the backward without its recompute
    return {
        "workload": f"{w.name}: kda_chunk_fwd_save then kda_chunk_bwd_saved (what the forward keeps "
                    f"feeds the backward; nothing recomputed), B={w.B}, T={w.T}, H={w.H}, d_k=d_v={w.dk}, "
                    "bf16 q/k/v/d_o",
        "value": w.tokens * world / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": ms, "steps": args.bwd_steps, "gpu_launches": launches * args.bwd_steps,
    }


def bench_decode(args, dev, world, rank, peaks, peak_kind):
    """kda_recurrent_step, ``--decode-steps`` consecutive steps on one state."""
    from gated_delta_rule_108_b200 import inputs as I
    from gated_delta_rule_108_b200 import kda

    w = I.workload(args.decode_workload)
    P = 8
    d = I.decode_inputs(dataclasses.replace(w, seed=w.seed + 1000 * rank), pool=P)
    g = {k: v.to(dev) for k, v in d.items()}
    st = g["state0"].clone()
    o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)
    steps = args.decode_steps
    for i in range(args.warmup):
        j = i % P
        kda.recurrent_step(g["q"][j], g["k"][j], g["v"][j], g["log_alpha"][j], g["beta"][j], st, o=o)
    st.copy_(g["state0"])
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
    dbytes = w.B * w.H * (2 * w.dk * w.dv * 4 + (2 * w.dk + 2 * w.dv) * 2 + 4 * w.dk + 4)
    dgbs = dbytes / (ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    tpu = traffic_per_unit("decode_step")
    return {
        "workload": f"{w.name}: kda_recurrent_step, B={w.B}, H={w.H}, d_k=d_v={w.dk}, bf16 q/k/v, "
                    f"fp32 state in place, {steps} consecutive steps (inputs cycle through {P} seeded draws)",
        "value": w.B * world / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": ms, "steps": steps, "gpu_launches": steps,
        "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": dgbs, "peak": hbm,
                     "unit": "GB/s", "frac": dgbs / hbm, "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": None if tpu is None else tpu * w.B * w.H,
                     "algorithmic_bytes_per_launch": dbytes, "ms_per_launch": ms},
    }


def bench_e2e(args, dev, world, res):
    """The headline forward through the public API from pinned host buffers:
    every step copies that step's inputs in and its outputs back.  Three
    streams pipeline the steps: the inputs of step i + 1 come in (copy engine)
    while step i computes and the outputs of step i - 1 go out (the other copy
    engine); device inputs and outputs are double-buffered."""
    from gated_delta_rule_108_b200 import kda

    x = res["x"]
    names = [n for n in ("q", "k", "v", "log_alpha", "beta", "initial_state", "cu_seqlens")
             if x[n] is not None]
    host = {n: x[n].pin_memory() for n in names}
    o, S, ws = res["o"], res["S"], res["ws"]
    devb = [{n: torch.empty_like(host[n], device=dev) for n in names} for _ in range(2)]
    outs = [(o, S), (torch.empty_like(o), torch.empty_like(S))]
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    S_h = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
    used = [False, False]

    def step(i):
        b = i & 1
        d, (ob, Sb) = devb[b], outs[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev["comp"][b])        # step i - 2 has read these inputs
            for n in names:
                d[n].copy_(host[n], non_blocking=True)
            ev["in"][b].record(s_in)
        comp.wait_event(ev["in"][b])
        if used[b]:
            comp.wait_event(ev["out"][b])             # step i - 2's outputs have gone out
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d.get("initial_state"),
                      d.get("cu_seqlens"), o=ob, final_state=Sb, workspace=ws)
        ev["comp"][b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            o_h.copy_(ob, non_blocking=True)
            S_h.copy_(Sb, non_blocking=True)
            ev["out"][b].record(s_out)
        used[b] = True

    steps = max(3, min(args.steps, 10))
    for i in range(min(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(comp)
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    for i in range(steps):
        step(i)
    comp.wait_stream(s_out)
    end.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world, dev) / steps
    return ms, h2d, d2h


def cpu_oracle_rate(w, x, heads, min_seconds=0.0, tokens=None):
    """Time the fp64 oracle on every sequence of ``x`` (its first ``tokens``
    tokens when given, fixed-length only) and the heads ``heads``, in whole
    passes repeated until ``min_seconds`` have gone by (at least one pass).
    Returns (tokens/s, seconds, passes, threads used); a token spans all w.H
    heads, so the sampled token-heads are divided by w.H."""
    from oracle import oracle as orc
    cu = x["cu_seqlens"]
    T = x["q"].shape[1] if tokens is None else tokens
    if cu is not None and tokens is not None:
        raise ValueError("a token prefix is only defined for fixed-length workloads")
    sl = {n: x[n][:, :T, heads].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    S0 = None if x["initial_state"] is None else x["initial_state"][:, heads].contiguous()
    n_heads = sl["q"].shape[2]
    token_heads = sl["q"].shape[0] * T * n_heads
    n_pairs = (sl["q"].shape[0] if cu is None else len(cu) - 1) * n_heads
    passes = 0
    t0 = time.perf_counter()
    while True:
        orc.kda_forward(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], S0, cu)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    return passes * token_heads / w.H / dt, dt, passes, min(orc.num_threads(), n_pairs)


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
    head = bench_chunk(args.workload, args.steps, args.warmup, dev, world, rank)
    extras = {}
    for name in [n for n in args.extra_workloads.split(",") if n and n != args.workload]:
        r = bench_chunk(name, args.steps, args.warmup, dev, world, rank)
        extras[name.lower()] = chunk_summary(r, world, peaks, peak_kind)
        del r
        torch.cuda.empty_cache()
    # the fused single pass (one CTA per (sequence, head), no intermediates in
    # memory), forced, beside the form kda_chunk_fwd picks by itself
    for name in [n for n in args.fused_workloads.split(",") if n]:
        old_path = os.environ.get("KDA_CHUNK_PATH")
        os.environ["KDA_CHUNK_PATH"] = "fused"
        try:
            r = bench_chunk(name, args.steps, args.warmup, dev, world, rank)
        finally:
            if old_path is None:
                os.environ.pop("KDA_CHUNK_PATH", None)
            else:
                os.environ["KDA_CHUNK_PATH"] = old_path
        summ_f = chunk_summary(r, world, peaks, peak_kind)
        summ_f["form"] = "fused single pass (forced; kernels_ms.intra_chunk is the whole pass)"
        summ_f["roofline"]["traffic"] = None   # the committed capture is of the split form's kernel
        extras[name.lower() + "_fused"] = summ_f
        del r
        torch.cuda.empty_cache()
    # fp32 inputs on the same shapes (split-tf32 tensor-core kernels)
    for name in [n for n in args.f32_workloads.split(",") if n]:
        r = bench_chunk(name, args.steps, args.warmup, dev, world, rank, dtype=torch.float32)
        summ_f = chunk_summary(r, world, peaks, peak_kind)
        summ_f["form"] = "two kernels, fp32 inputs: split-tf32 tensor-core products (3 MMAs each)"
        extras[name.lower() + "_f32"] = summ_f
        del r
        torch.cuda.empty_cache()
    dec = None if args.no_decode else bench_decode(args, dev, world, rank, peaks, peak_kind)
    bwd = None if args.no_bwd else bench_backward(args, dev, world, rank, peaks, peak_kind)
    train = None if (args.no_bwd or args.no_train) else bench_train(args, dev, world, rank)
    clk = clocks.stop()
    e2e = None if args.no_e2e else bench_e2e(args, dev, world, head)

    w = head["w"]
    summ = chunk_summary(head, world, peaks, peak_kind)
    from gated_delta_rule_108_b200 import kda as _kda
    plan = _kda.chunk_fwd_plan(w.B, w.T, w.H, w.dk, w.dv, w.num_seqs, w.lengths is not None, w.dtype)
    line = {
        "metric": METRIC,
        "value": summ["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": summ["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": data_recipe(w),
        "config": {
            "workload": describe(w),
            "global_batch": w.num_seqs * world,
            "seq_len": (f"{min(seq_lengths(w))}-{max(seq_lengths(w))} (packed, {w.tokens} tokens per rank)"
                        if w.lengths is not None else w.T),
            "heads": w.H,
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
            "l2": f"inputs larger than L2 ({method_bytes(w)['intra_chunk'] / 1e6:.0f} MB read per step)",
        },
        "roofline": summ["roofline"],
        "path_roofline": summ["path_roofline"],
        "kernels_ms": summ["kernels_ms"],
        "form": "fused single pass" if plan == 1 else "two kernels (intra-chunk, inter-chunk)",
        "chunk_head_items": summ["chunk_head_items"],
        "gpu_launches": head["launches"],
    }
    line.update(extras)
    if dec is not None:
        line["decode"] = dec
    if bwd is not None:
        line["chunk_bwd"] = bwd
    if train is not None:
        line["train_step"] = train
    if e2e is not None:
        ms_e, h2d, d2h = e2e
        line["e2e"] = {"value": w.tokens * world / (ms_e / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e,
                       "pipelining": "inputs of step i+1 in, step i computing, outputs of step i-1 out "
                                     "(three streams, double-buffered device buffers)"}
    if clk is not None:
        line["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads = slice(0, min(w.H, args.cpu_heads))
        rate, dt, passes, cores = cpu_oracle_rate(w, head["x"], heads, min_seconds=10.0)
        n_h = len(range(*heads.indices(w.H)))
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"every sequence of {w.name} ({w.tokens} tokens), heads 0-{n_h - 1} "
                                          f"of {w.H} ({passes} passes in {dt:.1f} s), fp64 C oracle, OpenMP "
                                          f"over (sequence, head); tokens/s = token-heads/s / {w.H}"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_check_launch(args):
    """The rank set-up alone, on CPU (gloo): rank 0 prints the world size that
    the line's n_gpus would report."""
    world, rank, _ = dist_setup(use_cuda=False)
    t = max_over_ranks(float(rank), world, torch.device("cpu"))
    if rank == 0:
        print(json.dumps({"n_gpus": world, "gpus_arg": args.gpus, "max_rank": t}), flush=True)
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
    # each step: sequence 0, all heads, its first --reference-tokens tokens
    n0 = seq_lengths(w)[0]
    tokens = min(args.reference_tokens, n0)
    a = 0 if x["cu_seqlens"] is None else int(x["cu_seqlens"][0])
    xs = {n: x[n][0:1, a:a + tokens].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    xs["initial_state"] = None if x["initial_state"] is None else x["initial_state"][0:1]
    xs["cu_seqlens"] = None
    del x
    heads = slice(0, w.H)
    for _ in range(args.warmup):
        cpu_oracle_rate(w, xs, heads)
    times = []
    cores = 1
    for _ in range(args.steps):
        _, dt, _, cores = cpu_oracle_rate(w, xs, heads)
        times.append(dt)
    ms = 1e3 * statistics.mean(times)
    value = tokens / (ms / 1e3)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": data_recipe(w),
        "config": {"workload": describe(w) + f"; each step = sequence 0, all heads, first {tokens} tokens",
                   "global_batch": w.num_seqs, "heads": w.H},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"sequence 0 of {w.num_seqs}, {w.H} heads, {tokens} tokens per step"},
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
    ap.add_argument("--workload", default="C4", help="headline chunk-forward workload (C0..C4 minus C3)")
    ap.add_argument("--extra-workloads", default="C1,C2", help="more chunk-forward workloads, comma-separated")
    ap.add_argument("--f32-workloads", default="C1",
                    help="chunk-forward workloads also timed with fp32 inputs (key <name>_f32)")
    ap.add_argument("--fused-workloads", default="C4",
                    help="chunk-forward workloads also timed with the fused single pass forced")
    ap.add_argument("--decode-workload", default="C3")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--bwd-workload", default="C1")
    ap.add_argument("--reference-tokens", type=int, default=1024)
    ap.add_argument("--cpu-heads", type=int, default=4, help="heads in the CPU-oracle sample")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward (kda_chunk_bwd) measurement")
    ap.add_argument("--bwd-steps", type=int, default=10)
    ap.add_argument("--no-train", action="store_true", help="skip the training-step (saved forward) measurement")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--check-launch", action="store_true",
                    help="set up the ranks only (CPU, gloo) and print the world size")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        raise SystemExit(relaunch_under_torchrun(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
    if args.check_launch:
        run_check_launch(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        log("note: fewer than 3 warm-up steps")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
