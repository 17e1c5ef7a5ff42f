"""Host-side helpers of bench.py on CPU: the timed oracle sample and the
DRAM-traffic lookup that only answers while the captured source is unchanged."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_108_b200 import inputs as I  # noqa: E402


def test_cpu_oracle_rate_repeats_whole_passes():
    w = I.workload("C0")
    x = I.chunk_inputs(w)
    rate, dt, passes, threads = bench.cpu_oracle_rate(w, x, slice(0, 1), min_seconds=0.2, tokens=128)
    assert dt >= 0.2 and passes >= 1
    assert threads >= 1
    # one of the H = 2 heads: token-heads / H
    assert rate == pytest.approx(passes * w.B * 128 * 1 / w.H / dt)
    # with no minimum, exactly one pass
    _, _, one, _ = bench.cpu_oracle_rate(w, x, slice(0, 2), tokens=128)
    assert one == 1


def test_cpu_oracle_rate_on_packed_sequences():
    lens = (70, 0, 33)
    w = I.ChunkWorkload("p", B=1, T=sum(lens), H=3, dk=64, dv=64, lengths=lens, seed=5)
    x = I.chunk_inputs(w)
    rate, dt, passes, threads = bench.cpu_oracle_rate(w, x, slice(0, 3))
    from oracle import oracle as orc
    assert passes == 1 and threads == min(orc.num_threads(), 3 * 3)   # 3 sequences x 3 heads
    assert rate == pytest.approx(sum(lens) / dt)


def test_workload_arithmetic():
    w = I.workload("C1")
    assert bench.chunk_units(w) == 4 * 64 * 16
    mb = bench.method_bytes(w)
    th = 4 * 4096 * 16
    assert mb["intra_chunk"] == th * 1284           # q, k, v bf16 + log_alpha fp32 + beta
    assert mb["inter_chunk"] == th * 256 + 2 * 4 * 16 * 128 * 128 * 4   # o + S0 read + final state
    assert bench.record_bytes_per_unit(w) == 74240
    c4 = I.workload("C4")
    assert bench.chunk_units(c4) == sum((n + 63) // 64 for n in c4.lengths) * 32
    c2 = I.workload("C2")   # zero initial state: only the final state is written
    assert bench.method_bytes(c2)["inter_chunk"] == 65536 * 32 * 256 + 32 * 128 * 128 * 4


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    table = {"k": {"source": "kernel.cu", "source_sha": sha, "bytes_per_unit": 1234}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_per_unit("k") == 1234
    assert bench.traffic_per_unit("other") is None
    src.write_text("__global__ void k() { /* changed */ }\n")   # counters no longer describe it
    assert bench.traffic_per_unit("k") is None


def test_committed_traffic_table_covers_the_reported_kernels():
    """Each kernel whose roofline the bench line reports has a committed capture,
    naming a source file that exists and a positive byte count."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for name in ("intra_chunk", "inter_chunk", "decode_step", "bwd_tc_products"):
        ent = table[name]
        assert os.path.exists(os.path.join(ROOT, ent["source"])), name
        assert len(ent["source_sha"]) == 16 and ent["bytes_per_unit"] > 0, name
