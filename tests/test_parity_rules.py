"""The acceptance helpers themselves (CPU)."""

import numpy as np

from tests import parity as PT


def test_bf16_half_ulp():
    assert PT.bf16_half_ulp(np.array([1.0]))[0] == 2 ** -8
    assert PT.bf16_half_ulp(np.array([1.99]))[0] == 2 ** -8
    assert PT.bf16_half_ulp(np.array([-2.5]))[0] == 2 ** -7
    assert PT.bf16_half_ulp(np.array([0.3]))[0] == 2 ** -10
