"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import numpy as np
import pytest

import pins
from oracle import oracle as orc


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


def test_decode_step_is_one_token_forward():
    """A decode step on B sequences equals B separate one-token forwards."""
    q, k, v, la, beta, S0 = pins.rand_problem(30, T=1, H=3, dk=5, dv=4, B=4)
    o, S = orc.kda_decode_step(q[:, 0], k[:, 0], v[:, 0], la[:, 0], beta[:, 0], S0)
    for b in range(4):
        ob, Sb = orc.kda_forward(q[b:b + 1], k[b:b + 1], v[b:b + 1], la[b:b + 1],
                                 beta[b:b + 1], S0[b:b + 1])
        np.testing.assert_array_equal(o[b], ob[0, 0])
        np.testing.assert_array_equal(S[b], Sb[0])


def test_rejects_bad_cu_seqlens():
    q, k, v, la, beta, _ = pins.rand_problem(31, T=8, H=1, dk=4, dv=4)
    with pytest.raises(ValueError):
        orc.kda_forward(q, k, v, la, beta, cu_seqlens=np.array([0, 5, 3, 8]))
    with pytest.raises(ValueError):
        orc.kda_forward(q, k, v, la, beta, cu_seqlens=np.array([0, 5, 7]))


def test_empty_sequence_keeps_state():
    rng = np.random.default_rng(32)
    S0 = rng.standard_normal((1, 2, 4, 3))
    z = np.zeros((1, 0, 2, 4))
    o, S = orc.kda_forward(z, z, np.zeros((1, 0, 2, 3)), z, np.zeros((1, 0, 2)), S0)
    assert o.shape == (1, 0, 2, 3)
    np.testing.assert_array_equal(S, S0)
