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
