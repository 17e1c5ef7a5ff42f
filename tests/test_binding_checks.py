"""The Python binding refuses tensors whose shapes disagree with the sizes the
kernels take from q (and v, cu_seqlens) before anything reaches the library:
such a tensor would be read or written out of bounds on the device.  CPU only:
the shape checks come before the device checks."""
import pytest
import torch

from gated_delta_rule_108_b200 import kda

B, T, H, DK, DV = 2, 10, 3, 64, 32


def fwd_args(**over):
    a = dict(q=torch.zeros(B, T, H, DK), k=torch.zeros(B, T, H, DK), v=torch.zeros(B, T, H, DV),
             log_alpha=torch.zeros(B, T, H, DK), beta=torch.zeros(B, T, H),
             initial_state=torch.zeros(B, H, DK, DV))
    a.update(over)
    return a


@pytest.mark.parametrize("name,bad", [
    ("k", torch.zeros(B, T, H, DV)),
    ("v", torch.zeros(B, T + 1, H, DV)),
    ("beta", torch.zeros(B, T, H, 1)),
    ("initial_state", torch.zeros(B + 1, H, DK, DV)),
    ("log_alpha", torch.zeros(B, T, H, DK + 1)),
])
def test_chunk_fwd_refuses_mismatched_inputs(name, bad):
    with pytest.raises(ValueError, match=name):
        kda.chunk_fwd(**fwd_args(**{name: bad}))


@pytest.mark.parametrize("name,bad", [
    ("o", torch.zeros(B, T, H, DK)),
    ("final_state", torch.zeros(B, H, DV, DK)),
])
def test_chunk_fwd_refuses_mismatched_outputs(name, bad):
    with pytest.raises(ValueError, match=name):
        kda.chunk_fwd(**fwd_args(), **{name: bad})


def test_chunk_fwd_varlen_rules():
    cu = torch.tensor([0, 4, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="B == 1"):
        kda.chunk_fwd(**fwd_args(), cu_seqlens=cu)
    one = fwd_args(q=torch.zeros(1, T, H, DK), k=torch.zeros(1, T, H, DK), v=torch.zeros(1, T, H, DV),
                   log_alpha=torch.zeros(1, T, H, DK), beta=torch.zeros(1, T, H),
                   initial_state=torch.zeros(3, H, DK, DV))
    with pytest.raises(ValueError, match="initial_state"):   # 2 sequences, 3 states
        kda.chunk_fwd(**one, cu_seqlens=cu)
    with pytest.raises(ValueError, match="cu_seqlens"):
        kda.chunk_fwd(**one, cu_seqlens=cu[None])
    with pytest.raises(ValueError, match="q must have 4"):
        kda.chunk_fwd(**fwd_args(q=torch.zeros(T, H, DK)))


def test_consistent_shapes_still_need_the_gpu():
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.chunk_fwd(**fwd_args())


@pytest.mark.parametrize("name,bad", [
    ("d_o", torch.zeros(B, T, H, DK)),
    ("d_final_state", torch.zeros(B, H, DK, DV + 1)),
])
def test_chunk_bwd_refuses_mismatched_cotangents(name, bad):
    a = fwd_args()
    d_o = torch.zeros(B, T, H, DV)
    kw = {"d_final_state": torch.zeros(B, H, DK, DV)}
    if name == "d_o":
        d_o = bad
    else:
        kw[name] = bad
    with pytest.raises(ValueError, match=name):
        kda.chunk_bwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], d_o,
                      initial_state=a["initial_state"], **kw)


@pytest.mark.parametrize("name,bad", [
    ("state", torch.zeros(B, H, DK, DV - 1)),
    ("beta", torch.zeros(B)),
    ("k", torch.zeros(B, H + 1, DK)),
    ("o", torch.zeros(B, H, DK)),
])
def test_recurrent_step_refuses_mismatched_tensors(name, bad):
    a = dict(q=torch.zeros(B, H, DK), k=torch.zeros(B, H, DK), v=torch.zeros(B, H, DV),
             log_alpha=torch.zeros(B, H, DK), beta=torch.zeros(B, H), state=torch.zeros(B, H, DK, DV))
    o = None
    if name == "o":
        o = bad
    else:
        a[name] = bad
    with pytest.raises(ValueError, match=name):
        kda.recurrent_step(**a, o=o)


def test_buffers_made_for_another_stream_are_marked_used_there(monkeypatch):
    """A buffer the binding allocates (on the current stream) for a call that
    runs on another stream is recorded on that stream, so the caching allocator
    does not hand its memory out again while the call may still use it."""
    class FakeStream:
        def __init__(self, handle):
            self.cuda_stream = handle

    class FakeTensor:
        def __init__(self):
            self.recorded = []

        def record_stream(self, s):
            self.recorded.append(s)

    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: FakeStream(1))
    side, same = FakeStream(2), FakeStream(1)
    a, b = FakeTensor(), FakeTensor()
    kda._used_on(side, "cuda:0", a, None, b)
    assert a.recorded == [side] and b.recorded == [side]
    c = FakeTensor()
    kda._used_on(same, "cuda:0", c)
    kda._used_on(None, "cuda:0", c)
    assert c.recorded == []
