"""The C-ABI library: it loads, exports every symbol include/kda.h declares, and
rejects bad arguments on the host (no GPU needed: nothing is launched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_108_b200 import build, kda
    build.build()
    return kda.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_recurrent_step", "kda_chunk_fwd_workspace_size",
              "kda_workspace_status", "kda_last_error", "kda_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in kda.h but not exported"


def test_version(lib):
    assert b"sm_100a" in lib.kda_version()


def test_workspace_size(lib):
    from gated_delta_rule_108_b200 import kda
    f32, bf16 = 0, 1
    s1 = lib.kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, bf16)
    assert s1 > 4 * 64 * 16 * 128 * 128  # at least the per-chunk records
    # varlen bound covers the fixed-length count for the same tokens
    s2 = lib.kda_chunk_fwd_workspace_size(1, 4 * 4096, 16, 128, 128, 4, 1, bf16)
    assert s2 >= s1
    assert lib.kda_chunk_fwd_workspace_size(1, 100, 2, 96, 64, 1, 0, f32) == 0  # unsupported dk
    assert lib.kda_chunk_fwd_workspace_size(2, 100, 2, 64, 64, 2, 1, f32) == 0  # varlen needs B=1
    assert kda.KDA_OK == 0


def _chunk(lib, **over):
    args = dict(q=1 << 20, k=1 << 20, v=1 << 20, la=1 << 20, beta=1 << 20, s0=None, cu=None,
                B=1, T=64, H=1, dk=64, dv=64, N=1, dtype=0, o=1 << 20, sf=None,
                ws=1 << 20, wsb=1 << 30, stream=None)
    args.update(over)
    a = args
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cu"],
                             a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dtype"],
                             a["o"], a["sf"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(dk=96), 2),                 # unsupported head size
    (dict(dtype=7), 1),               # unknown dtype
    (dict(q=None), 1),                # null input
    (dict(k=(1 << 20) + 4), 1),       # misaligned
    (dict(B=2, cu=1 << 20), 1),       # varlen with B != 1
    (dict(ws=None), 5),               # missing workspace
    (dict(ws=(1 << 20) + 16), 5),     # workspace not 256-aligned
    (dict(wsb=16), 5),                # workspace too small
    (dict(H=0), 1),
    (dict(s0=1 << 20, sf=(1 << 20) + 64), 1),  # partially overlapping states
])
def test_chunk_fwd_rejects(lib, over, status):
    assert _chunk(lib, **over) == status
    assert lib.kda_last_error()  # a message is set


def test_recurrent_step_rejects(lib):
    p = 1 << 20
    assert lib.kda_recurrent_step(p, p, p, p, p, p, 2, 2, 80, 64, 1, p + (1 << 24), None) == 2
    assert lib.kda_recurrent_step(None, p, p, p, p, p, 2, 2, 64, 64, 1, p + (1 << 24), None) == 1
    # o aliasing the state
    assert lib.kda_recurrent_step(p, p, p, p, p, p, 2, 2, 64, 64, 1, p, None) == 1


def test_python_binding_has_no_cpu_path(monkeypatch, tmp_path):
    """The binding raises when the library is missing instead of computing on the CPU."""
    from gated_delta_rule_108_b200 import kda
    monkeypatch.setenv("KDA_B200_LIB", str(tmp_path / "missing.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(kda.KDAError):
        kda.lib()


def test_gated_entry_points_validate(lib):
    p = 1 << 20
    f = lib.kda_chunk_fwd_gated
    # unknown gate kind
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 64, 64, 1, 0, 9, p, None, p, 1 << 30, None) == 1
    # a gate that needs log_alpha, given none
    assert f(p, p, p, None, p, None, None, 1, 64, 1, 64, 64, 1, 0, 0, p, None, p, 1 << 30, None) == 1
    assert f(p, p, p, None, p, None, None, 1, 64, 1, 64, 64, 1, 0, 1, p, None, p, 1 << 30, None) == 1
    # no gate: log_alpha may be NULL (fails later, on the missing workspace)
    assert f(p, p, p, None, p, None, None, 1, 64, 1, 64, 64, 1, 0, 2, p, None, None, 0, None) == 5
    # per-head gate: log_alpha only needs 4-byte alignment (fails on the workspace)
    assert f(p, p, p, p + 4, p, None, None, 1, 64, 1, 64, 64, 1, 0, 1, p, None, None, 0, None) == 5
    d = lib.kda_recurrent_step_gated
    assert d(p, p, p, None, p, p, 2, 2, 64, 64, 1, 0, p + (1 << 24), None) == 1
    assert d(p, p, p, p, p, p, 2, 2, 64, 64, 1, 7, p + (1 << 24), None) == 1


def _bwd(lib, **over):
    P = 1 << 20
    args = dict(q=P, k=P, v=P, la=P, beta=P, s0=None, cu=None, do=P, dsf=None,
                B=1, T=64, H=1, dk=64, dv=64, N=1, dtype=0, dq=P, dk_=P, dv_=P, dla=P, db=P,
                ds0=None, ws=P, wsb=1 << 30, stream=None)
    args.update(over)
    a = args
    return lib.kda_chunk_bwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cu"], a["do"],
                             a["dsf"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dtype"],
                             a["dq"], a["dk_"], a["dv_"], a["dla"], a["db"], a["ds0"], a["ws"],
                             a["wsb"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(dk=96), 2),                 # unsupported head size
    (dict(dtype=7), 1),               # unknown dtype
    (dict(do=None), 1),               # null cotangent
    (dict(la=None), 1),               # the backward takes the per-channel gate
    (dict(dla=None), 1),              # null gradient output
    (dict(v=(1 << 20) + 4), 1),       # misaligned
    (dict(B=2, cu=1 << 20), 1),       # varlen with B != 1
    (dict(ws=None), 5),               # missing workspace
    (dict(wsb=16), 5),                # workspace too small
    (dict(H=0), 1),
])
def test_chunk_bwd_rejects(lib, over, status):
    assert _bwd(lib, **over) == status
    assert lib.kda_last_error()


def lib_simt_record_bytes(dk, dv):
    """fp32 record bytes per (chunk, head): W, U0, Q~, K^, P, gamma, 256-byte padded."""
    floats = 64 * (3 * dk + dv + 64) + dk
    return (floats + 63) // 64 * 64 * 4


def test_bwd_workspace_size(lib):
    f32, bf16 = 0, 1
    fwd = lib.kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, f32)
    bwd = lib.kda_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, f32)
    units = 4 * 64 * 16
    # records + T + two state-sized buffers per (head, chunk) + dU
    assert bwd >= fwd + units * 4 * (64 * 64 + 2 * 128 * 128 + 64 * 128)
    # bf16 inputs: fp16 records (74,240 B per (chunk, head) at d = 128) instead of
    # fp32 ones, plus the value-side products (3 x 64 x 128 + 64 x 64 + 128 fp32)
    vs = 4 * (3 * 64 * 128 + 64 * 64 + 128)
    assert lib.kda_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, bf16) >= (
        bwd - units * lib_simt_record_bytes(128, 128) + units * (74240 + vs))
    assert lib.kda_chunk_bwd_workspace_size(1, 100, 2, 96, 64, 1, 0, f32) == 0


def test_debug_drop_copy_arms_and_disarms(lib):
    """The failure-path test hook: negative caps are rejected; arming and
    disarming need no GPU (the hook only takes effect in a bf16 chunk call)."""
    assert lib.kda_debug_drop_copy(-1) == 1
    assert lib.kda_debug_drop_copy(1000) == 0
    assert lib.kda_debug_drop_copy(0) == 0


def test_chunk_fwd_plan_without_a_device(lib, monkeypatch):
    bf16, f32 = 1, 0
    big = 1 << 40
    monkeypatch.delenv("KDA_CHUNK_PATH", raising=False)
    assert lib.kda_chunk_fwd_plan(1, 100, 2, 96, 64, 1, 0, bf16, big) == -1    # unsupported dk
    assert lib.kda_chunk_fwd_plan(4, 64, 8, 128, 128, 4, 0, f32, big) == 0      # fp32: split
    assert lib.kda_chunk_fwd_plan(4, 64, 8, 128, 128, 4, 0, bf16, big) == 0     # room for the records: split
    full = lib.kda_chunk_fwd_workspace_size(1, 300, 8, 128, 128, 3, 1, bf16)
    small = lib.kda_chunk_fwd_fused_workspace_size(1, 300, 8, 128, 128, 3, 1, bf16)
    assert 0 < small < full and small % 4 == 0
    assert lib.kda_chunk_fwd_fused_workspace_size(1, 300, 8, 128, 128, 3, 1, f32) == 0
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, bf16, full) == 0
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, bf16, small) == 1   # only the fused pass fits
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, bf16, small - 1) == -1
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, f32, small) == -1
    monkeypatch.setenv("KDA_CHUNK_PATH", "fused")
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, bf16, full) == 1
    monkeypatch.setenv("KDA_CHUNK_PATH", "split")
    assert lib.kda_chunk_fwd_plan(1, 300, 8, 128, 128, 3, 1, bf16, small) == -1


def test_saved_forward_entry_points_validate(lib):
    """kda_chunk_fwd_save needs the backward-sized workspace; kda_chunk_bwd_saved
    validates like kda_chunk_bwd.  (Every case fails before any launch.)"""
    p = 1 << 20
    f32 = 0
    fwd_bytes = lib.kda_chunk_fwd_workspace_size(1, 64, 1, 64, 64, 1, 0, f32)
    bwd_bytes = lib.kda_chunk_bwd_workspace_size(1, 64, 1, 64, 64, 1, 0, f32)
    assert bwd_bytes > fwd_bytes
    f = lib.kda_chunk_fwd_save
    # a forward-sized workspace is too small to keep what the backward needs
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 64, 64, 1, f32, 0, p, None, p, fwd_bytes, None) == 5
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 64, 64, 1, f32, 0, p, None, None, 0, None) == 5
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 64, 64, 1, f32, 9, p, None, p, bwd_bytes, None) == 1
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 96, 64, 1, f32, 0, p, None, p, bwd_bytes, None) == 2
    b = lib.kda_chunk_bwd_saved
    # null cotangent; workspace too small
    assert b(p, p, p, p, p, None, None, None, None, 1, 64, 1, 64, 64, 1, f32, 0,
             p, p, p, p, p, None, p, bwd_bytes, None) == 1
    assert b(p, p, p, p, p, None, None, p, None, 1, 64, 1, 64, 64, 1, f32, 0,
             p, p, p, p, p, None, p, 16, None) == 5
    # bf16: a workspace that would run the fused forward is still too small to save
    bf16 = 1
    fused_bytes = lib.kda_chunk_fwd_fused_workspace_size(1, 64, 1, 64, 64, 1, 0, bf16)
    assert fused_bytes > 0
    assert f(p, p, p, p, p, None, None, 1, 64, 1, 64, 64, 1, bf16, 0, p, None, p, fused_bytes, None) == 5
