"""The chunkwise (WY) algebra the kernels implement equals the token loop (fp64, CPU)."""
import numpy as np
import pytest

import pins
from chunk_algebra import chunked_head
from oracle import oracle as orc


@pytest.mark.parametrize("T,dk,dv,la_scale", [(64, 16, 8, 0.25), (200, 12, 20, 0.5), (130, 8, 8, 2.0),
                                               (1, 8, 8, 0.25), (65, 16, 16, 0.0)])
def test_chunked_equals_token_loop(T, dk, dv, la_scale):
    q, k, v, la, beta, S0 = pins.rand_problem(40 + T, T=T, H=1, dk=dk, dv=dv, la_scale=la_scale)
    o_ref, S_ref = orc.kda_forward(q, k, v, la, beta, S0)
    o, S = chunked_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0], S0[0, 0])
    scale_o = np.abs(o_ref).max()
    assert np.abs(o - o_ref[0, :, 0]).max() <= 1e-11 * max(scale_o, 1)
    assert np.abs(S - S_ref[0, 0]).max() <= 1e-11 * max(np.abs(S_ref).max(), 1)


def test_beta_edges_in_chunk():
    q, k, v, la, beta, S0 = pins.rand_problem(50, T=150, H=1, dk=8, dv=8)
    beta[0, ::3, 0] = 1.0
    beta[0, 1::3, 0] = 0.0
    o_ref, S_ref = orc.kda_forward(q, k, v, la, beta, S0)
    o, S = chunked_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0], S0[0, 0])
    assert np.abs(o - o_ref[0, :, 0]).max() < 1e-11
    assert np.abs(S - S_ref[0, 0]).max() < 1e-11


def _chunk(seed, L, dk=32, la_scale=0.5):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((L, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    q = rng.standard_normal((L, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    la = -np.exp(rng.standard_normal((L, dk))) * la_scale
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    return q, k, la, beta


@pytest.mark.parametrize("L", [64, 37, 1])
def test_mid_chunk_split_leaves_a_and_p_unchanged(L):
    """The kernels form A and P from k e^{g - g_m}, k e^{g_m - g}, q e^{g - g_m} with
    g_m the middle token's cumulative decay; the factor e^{g_m} cancels in every
    product, so A and P equal their unsplit definitions."""
    q, k, la, beta = _chunk(60 + L, L)
    g = np.cumsum(la, axis=0)
    gm = g[(L - 1) // 2]
    A_split = np.tril(beta[:, None] * ((k * np.exp(g - gm)) @ (k * np.exp(gm - g)).T), -1)
    P_split = np.tril((q * np.exp(g - gm)) @ (k * np.exp(gm - g)).T, 0)
    A_def = np.tril(beta[:, None] * ((k * np.exp(g)) @ (k * np.exp(-g)).T), -1)
    P_def = np.tril((q * np.exp(g)) @ (k * np.exp(-g)).T, 0)
    assert np.abs(A_split - A_def).max() <= 1e-12 * max(np.abs(A_def).max(), 1.0)
    assert np.abs(P_split - P_def).max() <= 1e-12 * max(np.abs(P_def).max(), 1.0)


@pytest.mark.parametrize("L", [64, 37, 16, 5])
def test_blocked_doubling_inverse_is_exact(L):
    """(I + A)^{-1} as the kernels form it -- exact 16 x 16 diagonal blocks, then
    T21 = -T22 A21 T11 for 16-row pairs and for the 32-row halves -- equals the
    inverse in fp64, also for a ragged chunk zero-padded to 64 rows."""
    import precision_model as pm
    q, k, la, beta = _chunk(80 + L, L)
    g = np.cumsum(la, axis=0)
    A = np.tril(beta[:, None] * ((k * np.exp(g)) @ (k * np.exp(-g)).T), -1)
    ref = np.linalg.inv(np.eye(L) + A)
    T = pm.inv_blocked(A, pm.ident)
    assert np.abs(T - ref).max() <= 1e-12 * np.abs(ref).max()
    Ap = np.zeros((64, 64))
    Ap[:L, :L] = A
    Tp = pm.inv_blocked(Ap, pm.ident)
    assert np.abs(Tp[:L, :L] - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.array_equal(Tp[L:, L:], np.eye(64 - L)) and not Tp[L:, :L].any() and not Tp[:L, L:].any()
    # the doubling step itself: [[T11, 0], [T21, T22]] inverts [[I + A11, 0], [A21, I + A22]]
    h = 32
    T11, T22 = np.linalg.inv(np.eye(h) + Ap[:h, :h]), np.linalg.inv(np.eye(h) + Ap[h:, h:])
    T21 = -T22 @ Ap[h:, :h] @ T11
    assert np.abs(np.block([[T11, np.zeros((h, h))], [T21, T22]]) - Tp).max() <= 1e-12 * np.abs(Tp).max()
