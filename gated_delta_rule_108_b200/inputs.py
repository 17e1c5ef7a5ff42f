"""Seeded synthetic inputs for the KDA hot path.

This module is shared by the CUDA path's tests and benchmark and by the fp64
oracle's tests.  It holds none of the recurrence's arithmetic: it only draws
random tensors and prepares them the way the workloads prescribe (unit-norm
q/k, sigmoid beta, negative log-decay), on the CPU with ``torch.Generator``.

Draw order per call is fixed: [lengths], q, k, v, beta, log_alpha, S0,
[beta edge-case permutation], all from one ``torch.Generator().manual_seed(seed)``.

Workloads (sizes and value distributions):

* ``C0``  chunk fwd, fp32, B=1, H=2, T=256, d=64, zero initial state.
* ``C1``  chunk fwd, bf16 q/k/v, B=4, H=16, T=4096, d=128, S0 ~ N(0, 0.01^2).
* ``C2``  chunk fwd, bf16, B=1, H=32, T=65536, d=128, slow decay
          log_alpha = -exp(N(0,1))/256, beta = sigmoid(N(1,1)), zero S0.
* ``C3``  decode, bf16, B=256, H=32, d=128, S0 ~ N(0, 0.01^2), 1024 steps.
* ``C4``  packed varlen chunk fwd, 16 sequences with lengths U[1024, 16384],
          H=32, d=128, bf16, S0 ~ N(0, 0.01^2) per sequence; 10% of tokens get
          beta = 1 exactly and a disjoint 10% beta = 0 exactly.

Common to all: q, k ~ N(0,1) then L2-normalised per token and head (in fp32,
before any bf16 rounding); v ~ N(0,1); beta = sigmoid(N(mu, 1)) per token and
head; log_alpha = -exp(N(0,1)) / div per token, head and key channel.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

CHUNK = 64


@dataclasses.dataclass(frozen=True)
class ChunkWorkload:
    """A chunk-forward workload: B x T tokens (or packed ``lengths``), H heads."""
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype = torch.bfloat16
    s0_std: float = 0.0          # 0 -> zero initial state
    la_div: float = 16.0         # log_alpha = -exp(N(0,1)) / la_div
    beta_mu: float = 0.0         # beta = sigmoid(N(beta_mu, 1))
    lengths: Optional[tuple] = None   # packed varlen sequence lengths (B must be 1)
    beta_edge_frac: float = 0.0  # fraction of tokens with beta := 1 and (disjoint) := 0
    seed: int = 0
    lengths_from: Optional[tuple] = None  # (n, lo, hi): lengths were drawn first from Generator(seed)

    @property
    def num_seqs(self) -> int:
        return len(self.lengths) if self.lengths is not None else self.B

    @property
    def tokens(self) -> int:
        """Total tokens (each token spans all H heads)."""
        return self.T if self.lengths is not None else self.B * self.T


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """A decode workload: B sequences x H heads, ``steps`` single-token steps."""
    name: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: torch.dtype = torch.bfloat16
    s0_std: float = 0.01
    la_div: float = 16.0
    beta_mu: float = 0.0
    seed: int = 3


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> tuple:
    """n sequence lengths uniform on [lo, hi] inclusive, from Generator(seed)."""
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


def _c4_lengths() -> tuple:
    return varlen_lengths(16, 1024, 16384, seed=4)


def workload(name: str):
    """The named workloads C0..C4 at their full sizes."""
    if name == "C0":
        return ChunkWorkload("C0", 1, 256, 2, 64, 64, torch.float32, 0.0, 16.0, 0.0, seed=0)
    if name == "C1":
        return ChunkWorkload("C1", 4, 4096, 16, 128, 128, torch.bfloat16, 0.01, 16.0, 0.0, seed=1)
    if name == "C2":
        return ChunkWorkload("C2", 1, 65536, 32, 128, 128, torch.bfloat16, 0.0, 256.0, 1.0, seed=2)
    if name == "C3":
        return DecodeWorkload("C3", 256, 32, 128, 128, 1024, torch.bfloat16, 0.01, 16.0, 0.0, seed=3)
    if name == "C4":
        lens = _c4_lengths()
        return ChunkWorkload("C4", 1, sum(lens), 32, 128, 128, torch.bfloat16, 0.01, 16.0,
                             0.0, lengths=lens, beta_edge_frac=0.1, seed=4,
                             lengths_from=(16, 1024, 16384))
    raise KeyError(name)


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def chunk_inputs(w: ChunkWorkload, heads: Optional[Sequence[int]] = None) -> dict:
    """Draw the inputs of a chunk-forward workload on the CPU.

    Returns a dict with q, k [B, T, H, dk] and v [B, T, H, dv] in ``w.dtype``,
    log_alpha [B, T, H, dk] fp32, beta [B, T, H] fp32, initial_state
    [N, H, dk, dv] fp32 (or None when s0_std == 0) and cu_seqlens (int32 [N+1],
    or None).  ``heads`` keeps only those heads after drawing the full tensors.
    """
    g = torch.Generator().manual_seed(w.seed)
    if w.lengths_from is not None:
        n, lo, hi = w.lengths_from
        drawn = tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))
        if drawn != tuple(w.lengths):
            raise ValueError("lengths do not match their recorded draw")
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    q = _unit(torch.randn(B, T, H, dk, generator=g))
    k = _unit(torch.randn(B, T, H, dk, generator=g))
    v = torch.randn(B, T, H, dv, generator=g)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g) + w.beta_mu)
    log_alpha = -torch.exp(torch.randn(B, T, H, dk, generator=g)) / w.la_div
    N = w.num_seqs
    S0 = None
    if w.s0_std > 0:
        S0 = torch.randn(N, H, dk, dv, generator=g) * w.s0_std
    if w.beta_edge_frac > 0:
        perm = torch.randperm(B * T, generator=g)
        n_edge = int(round(w.beta_edge_frac * B * T))
        flat = beta.view(B * T, H)
        flat[perm[:n_edge]] = 1.0
        flat[perm[n_edge:2 * n_edge]] = 0.0
    cu = None
    if w.lengths is not None:
        if B != 1:
            raise ValueError("packed varlen workloads need B == 1")
        cu = torch.zeros(len(w.lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(w.lengths, dtype=torch.int64), 0).to(torch.int32)
        assert int(cu[-1]) == T
    out = dict(q=q.to(w.dtype), k=k.to(w.dtype), v=v.to(w.dtype),
               log_alpha=log_alpha.float(), beta=beta.float(),
               initial_state=S0, cu_seqlens=cu)
    if heads is not None:
        hs = list(heads)
        for key in ("q", "k", "v", "log_alpha", "beta"):
            out[key] = out[key][:, :, hs].contiguous()
        if S0 is not None:
            out["initial_state"] = S0[:, hs].contiguous()
    return out


def decode_inputs(w: DecodeWorkload, pool: int) -> dict:
    """Draw a pool of ``pool`` distinct decode-step inputs plus the initial state.

    Step n of a run uses pool entry n % pool.  Returns q, k [P, B, H, dk],
    v [P, B, H, dv] in ``w.dtype``, log_alpha [P, B, H, dk] fp32, beta [P, B, H]
    fp32 and state0 [B, H, dk, dv] fp32.
    """
    g = torch.Generator().manual_seed(w.seed)
    P, B, H, dk, dv = pool, w.B, w.H, w.dk, w.dv
    q = _unit(torch.randn(P, B, H, dk, generator=g))
    k = _unit(torch.randn(P, B, H, dk, generator=g))
    v = torch.randn(P, B, H, dv, generator=g)
    beta = torch.sigmoid(torch.randn(P, B, H, generator=g) + w.beta_mu)
    log_alpha = -torch.exp(torch.randn(P, B, H, dk, generator=g)) / w.la_div
    S0 = torch.randn(B, H, dk, dv, generator=g) * w.s0_std
    return dict(q=q.to(w.dtype), k=k.to(w.dtype), v=v.to(w.dtype),
                log_alpha=log_alpha.float(), beta=beta.float(), state0=S0.float())
