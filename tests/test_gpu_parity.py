"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Tolerances (the accuracy bar of the workloads): fp32 inputs -> max relative
error ||g - r||_inf / ||r||_inf <= 1e-4; bf16 inputs -> relative L2 error
||g - r||_2 / ||r||_2 <= 5e-3, on o and on the final state, with the oracle run
in fp64 on the bf16-rounded inputs.  Full-size workloads are checked on every
(sequence, head) pair of C1, C2 and C4, each against its own oracle run.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_108_b200 import inputs as I
from gated_delta_rule_108_b200 import kda
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

TOL_F32_MAXREL = 1e-4
TOL_BF16_RELL2 = 5e-3


def rel_l2(g, r):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))


def max_rel(g, r):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


def check(g, r, dtype, what):
    g = g.float().cpu().numpy() if hasattr(g, "cpu") else g
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if dtype == torch.float32:
        e = max_rel(g, r)
        assert e <= TOL_F32_MAXREL, f"{what}: max rel error {e:.3e}"
    else:
        e = rel_l2(g, r)
        assert e <= TOL_BF16_RELL2, f"{what}: rel L2 error {e:.3e}"
    return e


def to_dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_chunk(x, **kw):
    g = to_dev(x)
    o, S = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                         g["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o, S


def oracle_chunk(x):
    return orc.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                           x["initial_state"], x["cu_seqlens"])


# ----------------------------------------------------------------- small ---
SHAPES = [(64, 64), (64, 128), (128, 64), (128, 128)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"dk{a}dv{b}" for a, b in SHAPES])
def test_chunk_fwd_small(cuda_device, dtype, dk, dv):
    # 3 full chunks and a ragged tail of 17 tokens, 2 sequences, 3 heads
    w = I.ChunkWorkload("small", B=2, T=209, H=3, dk=dk, dv=dv, dtype=dtype, s0_std=0.05, seed=21)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, dtype, "o")
    check(S, S_ref, dtype, "final_state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"dk{a}dv{b}" for a, b in SHAPES])
def test_recurrent_step_small(cuda_device, dtype, dk, dv):
    w = I.DecodeWorkload("small", B=5, H=3, dk=dk, dv=dv, steps=8, dtype=dtype, s0_std=0.1)
    d = I.decode_inputs(w, pool=8)
    st = d["state0"].cuda().clone()
    S_ref = d["state0"].double().numpy()
    for n in range(8):
        o = kda.recurrent_step(d["q"][n].cuda(), d["k"][n].cuda(), d["v"][n].cuda(),
                               d["log_alpha"][n].cuda(), d["beta"][n].cuda(), st)
        torch.cuda.synchronize()
        o_ref, S_ref = orc.kda_decode_step(d["q"][n], d["k"][n], d["v"][n], d["log_alpha"][n],
                                           d["beta"][n], S_ref)
        check(o, o_ref, dtype, f"o step {n}")
    check(st, S_ref, dtype, "state after 8 steps")


# ------------------------------------------------------------ full size ---
def test_c0_full(cuda_device):
    """fp32, B=1, H=2, T=256, d=64, zero initial state, seed 0: max rel <= 1e-4."""
    w = I.workload("C0")
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.float32, "C0 o")
    check(S, S_ref, torch.float32, "C0 final_state")


def _every_pair_check(name, head_group):
    """The whole workload in one call, then every (sequence, head) pair against
    the oracle (run on groups of ``head_group`` heads to bound host memory)."""
    w = I.workload(name)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o, S = o.cpu(), S.cpu()
    cu = x["cu_seqlens"]
    bounds = ([(s * w.T, (s + 1) * w.T) for s in range(w.B)] if cu is None
              else [(int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)])
    worst_o = worst_s = 0.0
    for h0 in range(0, w.H, head_group):
        hs = slice(h0, min(w.H, h0 + head_group))
        xs = {k: x[k][:, :, hs].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        S0 = None if x["initial_state"] is None else x["initial_state"][:, hs].contiguous()
        o_ref, S_ref = orc.kda_forward(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], S0, cu)
        o_g = o[:, :, hs].float().numpy()
        S_g = S[:, hs].numpy()
        if cu is None:   # [B, T, h, dv] -> [B*T, h, dv] token rows, like the packed layout
            o_g, o_ref = o_g.reshape(-1, *o_g.shape[2:]), o_ref.reshape(-1, *o_ref.shape[2:])
        else:
            o_g, o_ref = o_g[0], o_ref[0]
        for s, (a, b) in enumerate(bounds):
            for j in range(S_g.shape[1]):
                if b > a:
                    worst_o = max(worst_o, check(o_g[a:b, j], o_ref[a:b, j], w.dtype,
                                                 f"{name} o (seq {s}, head {h0 + j})"))
                worst_s = max(worst_s, check(S_g[s, j], S_ref[s, j], w.dtype,
                                             f"{name} final_state (seq {s}, head {h0 + j})"))
    return worst_o, worst_s


def test_c1_full_every_pair(cuda_device):
    """C1 (B=4, T=4096, H=16): all 64 (sequence, head) pairs."""
    _every_pair_check("C1", head_group=16)


def test_c2_full_every_head(cuda_device):
    """C2 (one 65,536-token sequence, H=32): all 32 heads."""
    _every_pair_check("C2", head_group=4)


def test_c4_varlen_full_every_pair(cuda_device):
    """C4 (16 packed sequences, about 147 k tokens, H=32): all 512 (sequence, head) pairs."""
    _every_pair_check("C4", head_group=4)


def test_c3_decode_full_sampled(cuda_device):
    """1024 steps, B=256, H=32; inputs cycle through a pool of 32 seeded draws."""
    w = I.workload("C3")
    P = 32
    d = I.decode_inputs(w, pool=P)
    g = {k: v.cuda() for k, v in d.items()}
    st = g["state0"].clone()
    o_last = None
    pairs = [(0, 0), (100, 17), (255, 31)]
    outs = {p: [] for p in pairs}
    for n in range(w.steps):
        j = n % P
        o_last = kda.recurrent_step(g["q"][j], g["k"][j], g["v"][j], g["log_alpha"][j],
                                    g["beta"][j], st)
        if n % 97 == 0 or n == w.steps - 1:
            oc = o_last.cpu()
            for (b, h) in pairs:
                outs[(b, h)].append((n, oc[b, h].clone()))
    torch.cuda.synchronize()
    S = st.cpu()
    idx = [n % P for n in range(w.steps)]
    for (b, h) in pairs:
        seq = {k: d[k][idx, b, h][None, :, None] for k in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, S_ref = orc.kda_forward(seq["q"], seq["k"], seq["v"], seq["log_alpha"], seq["beta"],
                                       d["state0"][b:b + 1, h:h + 1])
        got = torch.stack([t for _, t in outs[(b, h)]]).float().numpy()
        ref = np.stack([o_ref[0, n, 0] for n, _ in outs[(b, h)]])
        check(got, ref, w.dtype, f"C3 o (b {b}, h {h})")
        check(S[b:b + 1, h:h + 1], S_ref, w.dtype, f"C3 state (b {b}, h {h})")


@pytest.mark.parametrize("dk", [64, 128])
def test_many_chains_wide_slices(cuda_device, dk, monkeypatch):
    """Enough (sequence, head) chains that the two-kernel form's inter-chunk
    kernel takes whole 128-column value slices (one CTA per chain), with
    ragged sequences (the fused pass would take this input by itself)."""
    monkeypatch.setenv("KDA_CHUNK_PATH", "split")
    w = I.ChunkWorkload("wide", B=40, T=150, H=8, dk=dk, dv=128, dtype=torch.bfloat16, s0_std=0.05, seed=30)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o")
    check(S, S_ref, torch.bfloat16, "final_state")


# ----------------------------------------------------------- consistency ---
def test_chunk_equals_decode_steps(cuda_device):
    """The chunkwise and the recurrent modes agree on one sequence set."""
    w = I.ChunkWorkload("cons", B=3, T=130, H=2, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, seed=22)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    st = x["initial_state"].cuda().clone()
    g = to_dev(x)
    od = []
    for t in range(w.T):
        od.append(kda.recurrent_step(g["q"][:, t].contiguous(), g["k"][:, t].contiguous(),
                                     g["v"][:, t].contiguous(), g["log_alpha"][:, t].contiguous(),
                                     g["beta"][:, t].contiguous(), st))
    torch.cuda.synchronize()
    od = torch.stack(od, dim=1)
    assert rel_l2(od.float().cpu(), o.float().cpu()) < 5e-3
    assert rel_l2(st.cpu(), S.cpu()) < 5e-3
    o_ref, S_ref = oracle_chunk(x)
    check(od, o_ref, torch.bfloat16, "decode loop o")


def test_calls_on_a_side_stream(cuda_device):
    """Every call can run on a stream other than the current one; the buffers
    the binding allocates for it (o, states, gradients, workspace) stay
    reserved for that stream until its work is done."""
    w = I.ChunkWorkload("side", B=2, T=150, H=2, dk=128, dv=128, dtype=torch.bfloat16,
                        s0_std=0.05, seed=25)
    x = I.chunk_inputs(w)
    g = to_dev(x)
    cur, side = torch.cuda.current_stream(), torch.cuda.Stream()
    side.wait_stream(cur)   # the inputs were written on the current stream
    o, S = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["initial_state"],
                         stream=side)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "o")
    check(S, S_ref, torch.bfloat16, "final_state")

    d_o = torch.randn(o.shape, generator=torch.Generator().manual_seed(9)).to(o.dtype).cuda()
    side.wait_stream(cur)
    gs = kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o,
                       initial_state=g["initial_state"], stream=side)
    cur.wait_stream(side)
    gc = kda.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], d_o,
                       initial_state=g["initial_state"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        assert rel_l2(gs[n].float().cpu(), gc[n].float().cpu()) < 1e-5, n

    st_side, st_cur = S.clone(), S.clone()
    t = lambda a: a[:, 0].contiguous()
    side.wait_stream(cur)
    o_side = kda.recurrent_step(t(g["q"]), t(g["k"]), t(g["v"]), t(g["log_alpha"]), t(g["beta"]),
                                st_side, stream=side)
    cur.wait_stream(side)
    o_cur = kda.recurrent_step(t(g["q"]), t(g["k"]), t(g["v"]), t(g["log_alpha"]), t(g["beta"]), st_cur)
    torch.cuda.synchronize()
    assert rel_l2(o_side.float().cpu(), o_cur.float().cpu()) < 1e-6
    assert rel_l2(st_side.cpu(), st_cur.cpu()) < 1e-6


def test_split_sequence_carries_state(cuda_device):
    w = I.ChunkWorkload("split", B=2, T=300, H=2, dk=64, dv=128, dtype=torch.float32,
                        s0_std=0.05, seed=23)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    c = 100  # not a multiple of the chunk size
    xa = {k: (v[:, :c].contiguous() if k in ("q", "k", "v", "log_alpha", "beta") else v) for k, v in x.items()}
    oa, Sa = run_chunk(xa)
    xb = {k: (v[:, c:].contiguous() if k in ("q", "k", "v", "log_alpha", "beta") else v) for k, v in x.items()}
    xb["initial_state"] = Sa.cpu()
    ob, Sb = run_chunk(xb)
    assert max_rel(torch.cat([oa, ob], 1).cpu().numpy(), o.cpu().numpy()) < 1e-5
    assert max_rel(Sb.cpu().numpy(), S.cpu().numpy()) < 1e-5


def test_varlen_equals_separate_calls(cuda_device):
    lens = (1, 63, 64, 65, 0, 130, 200)
    w = I.ChunkWorkload("vl", B=1, T=sum(lens), H=2, dk=128, dv=64, dtype=torch.bfloat16,
                        s0_std=0.05, lengths=lens, beta_edge_frac=0.1, seed=24)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.bfloat16, "varlen o")
    check(S, S_ref, torch.bfloat16, "varlen final_state")
    cu = x["cu_seqlens"].tolist()
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        xs = {k: x[k][:, a:b].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        xs["initial_state"] = x["initial_state"][s:s + 1]
        xs["cu_seqlens"] = None
        os_, Ss = run_chunk(xs)
        assert torch.equal(os_.cpu(), o[:, a:b].cpu()), f"seq {s} o differs from the packed call"
        assert torch.equal(Ss.cpu(), S[s:s + 1].cpu()), f"seq {s} state differs from the packed call"


# ------------------------------------------------------------ edge cases ---
def test_empty_input_passes_state_through(cuda_device):
    S0 = torch.randn(2, 3, 64, 64).cuda()
    e = lambda *s: torch.empty(*s, device="cuda")
    q = e(2, 0, 3, 64).bfloat16()
    o, S = kda.chunk_fwd(q, q, e(2, 0, 3, 64).bfloat16(), e(2, 0, 3, 64), e(2, 0, 3), S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 3, 64) and torch.equal(S, S0)
    o, S = kda.chunk_fwd(q, q, e(2, 0, 3, 64).bfloat16(), e(2, 0, 3, 64), e(2, 0, 3), None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S) == 0


@pytest.mark.parametrize("case", ["beta0", "beta1", "nodecay"])
def test_degenerate_gates(cuda_device, case):
    w = I.ChunkWorkload("deg", B=1, T=150, H=2, dk=128, dv=128, dtype=torch.float32, s0_std=0.1, seed=25)
    x = I.chunk_inputs(w)
    if case == "beta0":
        x["beta"].zero_()
    elif case == "beta1":
        x["beta"].fill_(1.0)
    else:
        x["log_alpha"].zero_()
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, torch.float32, f"{case} o")
    check(S, S_ref, torch.float32, f"{case} final_state")


def test_state_alias_in_place(cuda_device):
    w = I.ChunkWorkload("alias", B=2, T=100, H=2, dk=64, dv=64, dtype=torch.bfloat16, s0_std=0.05, seed=26)
    x = I.chunk_inputs(w)
    o_ref, S_ref = oracle_chunk(x)
    g = to_dev(x)
    st = g["initial_state"].clone()
    o, S = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert S.data_ptr() == st.data_ptr()
    check(st, S_ref, torch.bfloat16, "aliased final_state")


def test_bad_cu_seqlens_reported(cuda_device):
    w = I.ChunkWorkload("bad", B=1, T=100, H=2, dk=64, dv=64, dtype=torch.bfloat16, seed=27)
    x = I.chunk_inputs(w)
    g = to_dev(x)
    cu = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device="cuda")  # decreasing
    o = torch.full((1, 100, 2, 64), 7.0, device="cuda").bfloat16()
    ws = torch.empty(kda.chunk_fwd_workspace_size(1, 100, 2, 64, 64, 3, True, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None, cu, o=o, workspace=ws)
    with pytest.raises(kda.KDAError) as ei:
        kda._check(kda.workspace_status(ws))
    assert ei.value.status == 6
    assert bool((o.float() == 7.0).all()), "o must be left unwritten"
    # a good call on the same workspace clears the status
    cu_ok = torch.tensor([0, 40, 60, 100], dtype=torch.int32, device="cuda")
    kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None, cu_ok, workspace=ws)
    assert kda.workspace_status(ws) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("where", ["all_channels", "few_channels"])
def test_strong_decay(cuda_device, dtype, where):
    """Chunks whose log-decay over half a chunk exceeds the split-factor range
    take the exact slow path for A and P; results still match the oracle."""
    w = I.ChunkWorkload("strong", B=2, T=200, H=2, dk=128, dv=64, dtype=dtype, s0_std=0.05, seed=28)
    x = I.chunk_inputs(w)
    g = torch.Generator().manual_seed(281)
    strong = -4.0 * torch.exp(0.2 * torch.randn(x["log_alpha"].shape, generator=g))
    if where == "all_channels":
        x["log_alpha"] = strong
    else:   # channels 5 and 77 of head 1 only
        x["log_alpha"][:, :, 1, [5, 77]] = strong[:, :, 1, [5, 77]]
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check(o, o_ref, dtype, f"{where} o")
    check(S, S_ref, dtype, f"{where} final_state")


@pytest.mark.parametrize("gate", ["channel", "head", "none"])
def test_f32_many_items_mixed_strong(cuda_device, gate):
    """fp32 inputs, persistent intra-chunk kernel with several (chunk, head) items per CTA:
    five packed sequences of ragged lengths (73 chunks) x H=12 = 876 items, d_k=128, d_v=64.
    With the per-channel gate, every third chunk of heads 0 and 5 decays strongly enough for
    the exact path; the per-head gate and no gate go to the oracle broadcast over the key
    channels.  Every (sequence, head) pair is checked."""
    lens = (1300, 1, 700, 64, 2477)
    w = I.ChunkWorkload("f32mix", B=1, T=sum(lens), H=12, dk=128, dv=64, dtype=torch.float32,
                        s0_std=0.05, lengths=lens, beta_edge_frac=0.1, seed=61)
    x = I.chunk_inputs(w)
    if gate == "channel":
        la = x["log_alpha"].clone()
        gen = torch.Generator().manual_seed(611)
        strong = (torch.arange(w.T) // 64) % 3 == 1
        for h in (0, 5):
            la[0, strong, h, :4] = -8.0 * torch.rand(int(strong.sum()), 4, generator=gen)
        x["log_alpha"] = la.contiguous()
    la_oracle = x["log_alpha"]
    if gate == "head":
        x["log_alpha"] = x["log_alpha"][..., 0].contiguous()
        la_oracle = x["log_alpha"][..., None].expand(la_oracle.shape).contiguous()
    elif gate == "none":
        x["log_alpha"] = None
        la_oracle = torch.zeros_like(la_oracle)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(dict(x, log_alpha=la_oracle))
    cu = x["cu_seqlens"].tolist()
    for s in range(len(lens)):
        for h in range(w.H):
            a, b = cu[s], cu[s + 1]
            if b > a:
                check(o[:, a:b, h], o_ref[:, a:b, h], torch.float32, f"{gate} seq {s} head {h} o")
            check(S[s, h], S_ref[s, h], torch.float32, f"{gate} seq {s} head {h} final_state")


@pytest.mark.parametrize("dk", [128, 64])
def test_f32_wide_slices(cuda_device, dk):
    """fp32 inputs with more (sequence, head) chains than 32-column slices fit in one wave
    (B=2, H=40, d_v=128: 80 chains x 4 > 148 SMs), so the inter-chunk kernel takes
    64-column slices (with d_k=128 one R3 buffer in tensor memory).  Every pair is checked."""
    w = I.ChunkWorkload("f32wide", B=2, T=300, H=40, dk=dk, dv=128, dtype=torch.float32, s0_std=0.05,
                        seed=62)
    x = I.chunk_inputs(w)
    o, S = run_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    for b in range(w.B):
        for h in range(w.H):
            check(o[b, :, h], o_ref[b, :, h], torch.float32, f"seq {b} head {h} o")
            check(S[b, h], S_ref[b, h], torch.float32, f"seq {b} head {h} final_state")


def test_value_range_reported(cuda_device):
    """bf16 path: a value beyond the fp16 range of the intermediates is reported."""
    w = I.ChunkWorkload("range", B=1, T=70, H=1, dk=64, dv=64, dtype=torch.bfloat16, seed=29)
    x = I.chunk_inputs(w)
    x["v"] = (x["v"].float() * 1e5).to(torch.bfloat16)
    g = to_dev(x)
    ws = torch.empty(kda.chunk_fwd_workspace_size(1, 70, 1, 64, 64, 1, False, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None, None, workspace=ws)
    assert kda.workspace_status(ws) == 7
