"""The hardware conversions the quantiser encodes with match their definitions
(E2M1 round-to-nearest-even on every float pattern, E4M3 on every non-negative
float, E2M1 stochastic rounding with the stated random-bit assignment on 2^28
pseudo-random pairs)."""

import pytest

from nvfp4_pretraining_linear_b200 import api

pytestmark = pytest.mark.gpu


def test_hardware_conversions_match_definitions():
    counts = api.check_conversions(n_sr=1 << 28)
    api.get_status()
    assert counts == [0, 0, 0], counts
