"""The fp64 oracle's backward against derivatives obtained another way (CPU only)."""
import numpy as np
import pytest

import pins_backward
from oracle import oracle as orc


@pytest.mark.parametrize("check", pins_backward.BACKWARD_CHECKS, ids=lambda c: c.__name__)
def test_backward_pin(check):
    check()


def test_backward_without_final_cotangent_equals_zero_cotangent():
    x, d_o, dSf, cu = pins_backward.rand_bwd_problem(76, (5, 7), H=1, dk=3, dv=3)
    a = orc.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                         initial_state=x["S0"], cu_seqlens=cu)
    b = orc.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                         initial_state=x["S0"], d_final_state=np.zeros_like(dSf), cu_seqlens=cu)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])


def test_backward_empty_sequence_passes_state_cotangent():
    """An empty sequence's dS0 is its final-state cotangent."""
    x, d_o, dSf, cu = pins_backward.rand_bwd_problem(77, (0, 4), H=2, dk=2, dv=3)
    g = orc.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o,
                         initial_state=x["S0"], d_final_state=dSf, cu_seqlens=cu)
    np.testing.assert_array_equal(g["dS0"][0], dSf[0])
