"""Checks that pin the fp64 oracle to what the pages and the mathematics fix.

Each ``check_*`` function runs the oracle (optionally a given compiled copy,
``lib``) on a small fp64 problem and raises ``AssertionError`` if the result
disagrees with something other than the oracle itself: a hand-derived worked
example, a closed form, an invariant stated on the pages, a reduction to a
simpler method written in another page's notation, the explicit matrix form of
the update, a gradient computed by autograd, or linearity.

Page references:
  [P3] daiw.net "Kimi Delta Attention" -- section "KDA 的更新式" (the update
       equation), its sub-sections on Diag(alpha_t), on I - beta k k^T, and on
       the DPLR structure; "同一个 key 被反复写入时不会无限累积".
  [P4] news.bugfactory.tech/news/3610 -- the DeltaNet paragraph (predict with
       the same key, error times beta, write the error; beta = 1 recalls the
       target exactly; orthogonal directions unchanged; one gradient step on the
       squared error), the Gated DeltaNet paragraph (scalar gate applied before
       predicting, order matters), and the KDA paragraph (per-channel gate,
       transition D_t - beta_t D_t k k^T, read with d_k^{-1/2}).
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_problem(seed, T=24, H=2, dk=8, dv=6, B=1, s0=True, la_scale=0.25):
    """Random fp64 problem: unit q/k, beta in (0,1), log_alpha < 0."""
    rng = np.random.default_rng(seed)
    q = _unit(rng.standard_normal((B, T, H, dk)))
    k = _unit(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    la = -np.exp(rng.standard_normal((B, T, H, dk))) * la_scale
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, la, beta, S0


def _close(a, b, tol, what):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol, f"{what}: max abs error {err:.3e} > {tol:.1e}"
    return err


def check_golden(lib=None):
    """Hand-derived two-token example (tests/golden/kda_worked_example_2x2.json)."""
    with open(os.path.join(GOLDEN, "kda_worked_example_2x2.json")) as f:
        g = json.load(f)
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    la = np.log(np.array(g["alpha"]))[None, :, None, :]
    beta = np.array(g["beta"])[None, :, None]
    S0 = np.array(g["initial_state"])[None, None]
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    tol = g["tolerance_abs"]
    _close(o[0, :, 0, :], np.array(g["expected_o"]), tol, "golden o")
    _close(S[0, 0], np.array(g["expected_final_state"]), tol, "golden final_state")


def check_exact_recall(lib=None):
    """[P4] beta = 1 and a unit key: querying that key returns v_t at once.

    With q_t = k_t the output is d_k^{-1/2} v_t for every token, whatever the
    state and the decay were.
    """
    q, k, v, la, beta, S0 = rand_problem(1, T=20, dk=8, dv=5)
    beta[:] = 1.0
    o, _ = orc.kda_forward(k, k, v, la, beta, S0, lib=lib)
    _close(o, v / np.sqrt(k.shape[-1]), 1e-12, "exact recall")


def check_orthogonal_directions(lib=None):
    """[P4] directions orthogonal to k_t are left alone, apart from the decay.

    For x with <x, k_t> = 0:  S_t^T x = S_{t-1}^T (alpha_t * x).
    """
    q, k, v, la, beta, S0 = rand_problem(2, T=9, H=1, dk=7, dv=4)
    _, S_prev = orc.kda_forward(q[:, :-1], k[:, :-1], v[:, :-1], la[:, :-1], beta[:, :-1], S0, lib=lib)
    _, S_t = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    rng = np.random.default_rng(20)
    kt = k[0, -1, 0]
    alpha = np.exp(la[0, -1, 0])
    for _ in range(4):
        x = rng.standard_normal(kt.shape)
        x -= (x @ kt) * kt
        _close(S_t[0, 0].T @ x, S_prev[0, 0].T @ (alpha * x), 1e-12, "orthogonal direction")


def _deltanet_ket(q, k, v, beta, S0_ket, gate=None):
    """DeltaNet / Gated DeltaNet in [P4]'s ket notation, S in R^{dv x dk}.

    S~ = a_t S (scalar gate, Gated DeltaNet; a_t = 1 for DeltaNet);
    v^ = S~ k; e = beta (v - v^); S = S~ + e k^T; o = d_k^{-1/2} S q.
    """
    T, dk = k.shape
    S = S0_ket.copy()
    out = []
    for t in range(T):
        if gate is not None:
            S = gate[t] * S
        vhat = S @ k[t]
        e = beta[t] * (v[t] - vhat)
        S = S + np.outer(e, k[t])
        out.append(S @ q[t] / np.sqrt(dk))
    return np.array(out), S


def check_deltanet_reduction(lib=None):
    """[P4]/[P3]: with alpha = 1 (log_alpha = 0) KDA is DeltaNet."""
    q, k, v, la, beta, S0 = rand_problem(3, T=30, H=2, dk=6, dv=5)
    la[:] = 0.0
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    for h in range(q.shape[2]):
        o_ref, S_ref = _deltanet_ket(q[0, :, h], k[0, :, h], v[0, :, h], beta[0, :, h], S0[0, h].T)
        _close(o[0, :, h], o_ref, 1e-12, "DeltaNet o")
        _close(S[0, h], S_ref.T, 1e-12, "DeltaNet state")


def check_gated_deltanet_reduction(lib=None):
    """[P4]/[P3]: one decay shared by all channels gives Gated DeltaNet."""
    q, k, v, la, beta, S0 = rand_problem(4, T=30, H=2, dk=6, dv=5)
    la[:] = la[..., :1]  # same value in every key channel
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    for h in range(q.shape[2]):
        gate = np.exp(la[0, :, h, 0])
        o_ref, S_ref = _deltanet_ket(q[0, :, h], k[0, :, h], v[0, :, h], beta[0, :, h],
                                     S0[0, h].T, gate=gate)
        _close(o[0, :, h], o_ref, 1e-12, "Gated DeltaNet o")
        _close(S[0, h], S_ref.T, 1e-12, "Gated DeltaNet state")


def check_beta_zero(lib=None):
    """beta = 0 leaves only the channel-wise decay: a closed form.

    S_t = Diag(exp(sum_{j<=t} log_alpha_j)) S_0 and o_t = d_k^{-1/2} S_t^T q_t.
    """
    q, k, v, la, beta, S0 = rand_problem(5, T=17, H=2, dk=5, dv=4)
    beta[:] = 0.0
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    g = np.cumsum(la, axis=1)  # [B, T, H, dk]
    for h in range(2):
        for t in range(q.shape[1]):
            St = np.exp(g[0, t, h])[:, None] * S0[0, h]
            _close(o[0, t, h], St.T @ q[0, t, h] / np.sqrt(5), 1e-12, "beta=0 output")
        _close(S[0, h], np.exp(g[0, -1, h])[:, None] * S0[0, h], 1e-12, "beta=0 state")


def check_orthonormal_keys(lib=None):
    """[P3] no accumulation on re-write; orthonormal keys store exactly.

    beta = 1, alpha = 1, S_0 = 0 and orthonormal keys k_1..k_m give
    S_m = sum_i k_i v_i^T.  Writing the same key twice keeps only the last value.
    """
    rng = np.random.default_rng(6)
    dk, dv, m = 8, 3, 6
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q[:, :m].T  # m orthonormal rows
    v = rng.standard_normal((m, dv))
    shp = lambda a: a[None, :, None, :]
    ones = np.ones((1, m, 1))
    _, S = orc.kda_forward(shp(keys), shp(keys), shp(v), np.zeros((1, m, 1, dk)), ones, lib=lib)
    _close(S[0, 0], keys.T @ v, 1e-12, "orthonormal keys")
    # the same key written twice: the first value is fully replaced
    kk = np.stack([keys[0], keys[0]])
    vv = rng.standard_normal((2, dv))
    _, S2 = orc.kda_forward(shp(kk), shp(kk), shp(vv), np.zeros((1, 2, 1, dk)), np.ones((1, 2, 1)), lib=lib)
    _close(S2[0, 0], np.outer(keys[0], vv[1]), 1e-12, "re-write of one key")


def check_unrolled_matrix_form(lib=None):
    """[P3] the update equation as explicit d_k x d_k matrix products, unrolled.

    M_j = (I - beta_j k_j k_j^T) Diag(alpha_j);
    S_t = (M_t ... M_1) S_0 + sum_{i<=t} (M_t ... M_{i+1}) beta_i k_i v_i^T,
    o_t = d_k^{-1/2} S_t^T q_t, by brute force for T <= 16.
    """
    q, k, v, la, beta, S0 = rand_problem(7, T=16, H=1, dk=5, dv=3)
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    T, dk = q.shape[1], q.shape[3]
    I = np.eye(dk)
    M = [(I - beta[0, j, 0] * np.outer(k[0, j, 0], k[0, j, 0])) @ np.diag(np.exp(la[0, j, 0]))
         for j in range(T)]

    def phi(t, i):  # M_t M_{t-1} ... M_{i+1}  (0-based tokens: product over j in (i, t])
        P = I.copy()
        for j in range(i + 1, t + 1):
            P = M[j] @ P
        return P

    for t in range(T):
        St = phi(t, -1) @ S0[0, 0]
        for i in range(t + 1):
            St = St + phi(t, i) @ (beta[0, i, 0] * np.outer(k[0, i, 0], v[0, i, 0]))
        _close(o[0, t, 0], St.T @ q[0, t, 0] / np.sqrt(dk), 1e-11, "unrolled o")
    _close(S[0, 0], St, 1e-11, "unrolled state")


def check_dplr_ket_form(lib=None):
    """[P4] ket form with the DPLR transition A_t = D_t - beta_t D_t k k^T.

    S (d_v x d_k) evolves as S_t = S_{t-1} A_t + beta_t v_t k_t^T,
    o_t = d_k^{-1/2} S_t q_t.
    """
    q, k, v, la, beta, S0 = rand_problem(8, T=25, H=1, dk=6, dv=4)
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    Sk = S0[0, 0].T.copy()
    for t in range(q.shape[1]):
        D = np.diag(np.exp(la[0, t, 0]))
        kt = k[0, t, 0]
        A = D - beta[0, t, 0] * D @ np.outer(kt, kt)
        Sk = Sk @ A + beta[0, t, 0] * np.outer(v[0, t, 0], kt)
        _close(o[0, t, 0], Sk @ q[0, t, 0] / np.sqrt(6), 1e-12, "DPLR ket o")
    _close(S[0, 0], Sk.T, 1e-12, "DPLR ket state")


def check_gradient_step(lib=None):
    """[P4] the delta update is one gradient step of size beta on the squared error.

    With S~ = Diag(alpha_t) S_{t-1} and L(S) = 1/2 ||S^T k_t - v_t||^2:
    S_t = S~ - beta_t dL/dS (S~); the gradient comes from torch autograd.
    """
    import torch

    q, k, v, la, beta, S0 = rand_problem(9, T=6, H=1, dk=5, dv=4)
    _, S_prev = orc.kda_forward(q[:, :-1], k[:, :-1], v[:, :-1], la[:, :-1], beta[:, :-1], S0, lib=lib)
    _, S_t = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    St = torch.tensor(np.exp(la[0, -1, 0])[:, None] * S_prev[0, 0], dtype=torch.float64,
                      requires_grad=True)
    kt = torch.tensor(k[0, -1, 0])
    vt = torch.tensor(v[0, -1, 0])
    loss = 0.5 * ((St.T @ kt - vt) ** 2).sum()
    (grad,) = torch.autograd.grad(loss, St)
    expect = (St - beta[0, -1, 0] * grad).detach().numpy()
    _close(S_t[0, 0], expect, 1e-12, "gradient step")


def check_linearity(lib=None):
    """For fixed q, k, alpha, beta the map (S_0, V) -> (o, S_T) is linear."""
    q, k, v, la, beta, S0 = rand_problem(10, T=20, H=2, dk=6, dv=5)
    rng = np.random.default_rng(11)
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    a, b = 0.7, -1.3
    o1, S1 = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    o2, S2 = orc.kda_forward(q, k, v2, la, beta, S02, lib=lib)
    o3, S3 = orc.kda_forward(q, k, a * v + b * v2, la, beta, a * S0 + b * S02, lib=lib)
    _close(o3, a * o1 + b * o2, 1e-11, "linearity o")
    _close(S3, a * S1 + b * S2, 1e-11, "linearity state")


def check_split_sequence(lib=None):
    """The final state is the whole recurrence: running two halves with the
    state carried across equals one run over the whole sequence."""
    q, k, v, la, beta, S0 = rand_problem(12, T=40, H=2, dk=6, dv=5, B=2)
    o, S = orc.kda_forward(q, k, v, la, beta, S0, lib=lib)
    c = 17
    oa, Sa = orc.kda_forward(q[:, :c], k[:, :c], v[:, :c], la[:, :c], beta[:, :c], S0, lib=lib)
    ob, Sb = orc.kda_forward(q[:, c:], k[:, c:], v[:, c:], la[:, c:], beta[:, c:], Sa, lib=lib)
    _close(np.concatenate([oa, ob], axis=1), o, 1e-12, "split o")
    _close(Sb, S, 1e-12, "split state")


def check_varlen_packing(lib=None):
    """Packed sequences (cu_seqlens) equal separate runs, including empty ones."""
    lens = [5, 0, 13, 1, 9]
    T = sum(lens)
    q, k, v, la, beta, _ = rand_problem(13, T=T, H=2, dk=4, dv=3)
    rng = np.random.default_rng(14)
    S0 = rng.standard_normal((len(lens), 2, 4, 3))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, S = orc.kda_forward(q, k, v, la, beta, S0, cu_seqlens=cu, lib=lib)
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        sl = slice(a, b)
        os_, Ss = orc.kda_forward(q[:, sl], k[:, sl], v[:, sl], la[:, sl], beta[:, sl],
                                  S0[s:s + 1], lib=lib)
        _close(o[:, sl], os_, 0.0, f"varlen o seq {s}")
        _close(S[s], Ss[0], 0.0, f"varlen state seq {s}")


ALL_CHECKS = [
    check_golden,
    check_exact_recall,
    check_orthogonal_directions,
    check_deltanet_reduction,
    check_gated_deltanet_reduction,
    check_beta_zero,
    check_orthonormal_keys,
    check_unrolled_matrix_form,
    check_dplr_ket_form,
    check_gradient_step,
    check_linearity,
    check_split_sequence,
    check_varlen_packing,
]
