"""Host-side logic of the N-rank benchmark on CPU: gloo, world size 2."""
import json
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from gated_delta_rule_108_b200 import inputs as I
    # every rank ends with the slowest rank's time
    t = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
    # each rank draws its own batch (weak scaling): different seeds -> different data
    w = I.workload("C0")
    wr = I.ChunkWorkload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    x = I.chunk_inputs(wr)
    qsum = torch.tensor([float(x["q"].double().sum())])
    gathered = [torch.zeros(1) for _ in range(world)]
    dist.all_gather(gathered, qsum)
    q.put((rank, t, [float(g) for g in gathered]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, sums in out:
        assert t == 11.0
        assert sums[0] != sums[1]


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_gpus_flag_starts_that_many_ranks():
    """bench.py --gpus 2 outside torchrun relaunches itself as two ranks; the
    line's n_gpus is the world size those ranks see (CPU, gloo)."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--check-launch"],
                       env=env, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["gpus_arg"] == 2 and out["max_rank"] == 1.0


def test_gpus_flag_must_match_world_size():
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4", "--check-launch"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE=2" in r.stderr
