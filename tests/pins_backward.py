"""Checks that pin the fp64 oracle's backward (``kda_backward``) to something
other than itself.

The backward is the reverse-mode derivative of the token recurrence (daiw.net
"Kimi Delta Attention", section "KDA 的更新式"; the chunkwise training mode of
news.bugfactory.tech/news/3610, KDA paragraph).  Its gradients are fixed by the
forward alone, so each check compares them with a derivative obtained another
way:

* central finite differences of the fp64 forward oracle, element by element,
  on tiny packed problems, one of them long enough to cross the backward's
  recomputation segments;
* exact directional derivatives: the loss <d_o, o> + <dS_T, S_T> is linear in
  q, and jointly linear in (v, S0), so a finite step of any size along those
  directions changes it by exactly <gradient, step>;
* torch autograd through an independently written matrix form of the update,
  S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.

Each ``check_*`` takes an optional compiled oracle ``lib`` so that planted
mistakes can be run against them.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as orc

NAMES = ("q", "k", "v", "log_alpha", "beta", "S0")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def rand_bwd_problem(seed, lengths, H, dk, dv, la_scale=0.3):
    """Packed fp64 problem with cotangents for o and the final state."""
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    N = len(lengths)
    x = {
        "q": rng.standard_normal((1, T, H, dk)) / np.sqrt(dk),
        "k": rng.standard_normal((1, T, H, dk)) / np.sqrt(dk),
        "v": rng.standard_normal((1, T, H, dv)),
        "log_alpha": -np.exp(rng.standard_normal((1, T, H, dk))) * la_scale,
        "beta": 1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, H)))),
        "S0": rng.standard_normal((N, H, dk, dv)) * 0.5,
    }
    d_o = rng.standard_normal((1, T, H, dv))
    dSf = rng.standard_normal((N, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return x, d_o, dSf, cu


def _loss(x, d_o, dSf, cu, lib):
    o, S = orc.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                           cu_seqlens=cu, lib=lib)
    return float(np.sum(o * d_o) + np.sum(S * dSf))


def _grads(x, d_o, dSf, cu, lib):
    return orc.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                            initial_state=x["S0"], d_final_state=dSf, cu_seqlens=cu, lib=lib)


def _fd_compare(x, d_o, dSf, cu, g, picks, lib, eps=1e-6, rtol=1e-6):
    """Central differences at the chosen (name, flat index) entries."""
    scale = 1.0 + max(float(np.max(np.abs(g[n]))) for n in GRADS if g[n].size)
    for name, idx in picks:
        xp = {n: a.copy() for n, a in x.items()}
        xm = {n: a.copy() for n, a in x.items()}
        xp[name].flat[idx] += eps
        xm[name].flat[idx] -= eps
        fd = (_loss(xp, d_o, dSf, cu, lib) - _loss(xm, d_o, dSf, cu, lib)) / (2 * eps)
        an = g[GRADS[NAMES.index(name)]].flat[idx]
        assert abs(fd - an) <= rtol * scale, (
            f"d{name}[{np.unravel_index(idx, x[name].shape)}]: backward {an:.10e}, "
            f"finite difference {fd:.10e}")


def check_bwd_finite_differences(lib=None):
    """Every gradient entry of a tiny packed problem (lengths 3, 0, 6) against
    central differences of the forward."""
    x, d_o, dSf, cu = rand_bwd_problem(70, (3, 0, 6), H=2, dk=3, dv=2)
    g = _grads(x, d_o, dSf, cu, lib)
    picks = [(n, i) for n in NAMES for i in range(x[n].size)]
    _fd_compare(x, d_o, dSf, cu, g, picks, lib)


def check_bwd_finite_differences_long(lib=None):
    """A 150-token sequence (three recomputation segments of the backward) and a
    short one: tokens on both sides of every segment edge and a random sample."""
    x, d_o, dSf, cu = rand_bwd_problem(71, (150, 5), H=1, dk=3, dv=2, la_scale=0.05)
    g = _grads(x, d_o, dSf, cu, lib)
    rng = np.random.default_rng(72)
    picks = []
    for name in NAMES[:5]:
        shp = x[name].shape
        toks = [0, 1, 62, 63, 64, 65, 126, 127, 128, 129, 149, 150, 154]
        toks += list(rng.integers(0, shp[1], 6))
        for t in toks:
            inner = int(rng.integers(0, int(np.prod(shp[2:]))))
            picks.append((name, t * int(np.prod(shp[2:])) + inner))
    picks += [("S0", i) for i in range(x["S0"].size)]
    _fd_compare(x, d_o, dSf, cu, g, picks, lib)


def check_bwd_linear_directions(lib=None):
    """Finite steps along q, and along (v, S0) together, change the loss by
    exactly <gradient, step> (the loss is linear in those inputs)."""
    x, d_o, dSf, cu = rand_bwd_problem(73, (40, 90), H=2, dk=5, dv=4)
    g = _grads(x, d_o, dSf, cu, lib)
    rng = np.random.default_rng(74)
    L0 = _loss(x, d_o, dSf, cu, lib)
    for names in (("q",), ("v", "S0")):
        y = {n: a.copy() for n, a in x.items()}
        pred = 0.0
        for n in names:
            step = rng.standard_normal(x[n].shape)
            y[n] = x[n] + step
            pred += float(np.sum(g[GRADS[NAMES.index(n)]] * step))
        dL = _loss(y, d_o, dSf, cu, lib) - L0
        assert abs(dL - pred) <= 1e-9 * (1.0 + abs(pred)), f"{names}: dL {dL:.12e} vs {pred:.12e}"


def _torch_matrix_form(q, k, v, la, beta, S0, cu):
    """S_t = (I - beta k k^T) Diag(exp(la)) S_{t-1} + beta k v^T;  o_t = S_t^T q_t / sqrt(dk)."""
    _, T, H, dk = q.shape
    outs, finals = [], []
    eye = torch.eye(dk, dtype=q.dtype)
    for s in range(len(cu) - 1):
        heads_o, heads_S = [], []
        for h in range(H):
            S = S0[s, h]
            rows = []
            for t in range(int(cu[s]), int(cu[s + 1])):
                kt = k[0, t, h][:, None]
                M = (eye - beta[0, t, h] * (kt @ kt.T)) @ torch.diag(torch.exp(la[0, t, h]))
                S = M @ S + beta[0, t, h] * kt @ v[0, t, h][None, :]
                rows.append(S.T @ q[0, t, h] / dk ** 0.5)
            heads_o.append(torch.stack(rows) if rows else torch.zeros(0, S.shape[1], dtype=q.dtype))
            heads_S.append(S)
        outs.append(torch.stack(heads_o, 1))
        finals.append(torch.stack(heads_S))
    return torch.cat(outs, 0)[None], torch.stack(finals)


def check_bwd_autograd(lib=None):
    """All six gradients against torch autograd of the matrix form (two packed
    sequences, one crossing a recomputation segment edge)."""
    x, d_o, dSf, cu = rand_bwd_problem(75, (70, 9), H=2, dk=4, dv=3)
    g = _grads(x, d_o, dSf, cu, lib)
    t = {n: torch.tensor(a, requires_grad=True) for n, a in x.items()}
    o, S = _torch_matrix_form(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["S0"], cu)
    loss = (o * torch.tensor(d_o)).sum() + (S * torch.tensor(dSf)).sum()
    loss.backward()
    for n, gn in zip(NAMES, GRADS):
        ref = t[n].grad.numpy()
        err = float(np.max(np.abs(ref - g[gn])))
        assert err <= 1e-10 * (1.0 + float(np.max(np.abs(ref)))), f"{gn}: max abs error {err:.3e}"


BACKWARD_CHECKS = [
    check_bwd_finite_differences,
    check_bwd_finite_differences_long,
    check_bwd_linear_directions,
    check_bwd_autograd,
]
