"""The oracle's V2 Target Scale-Up layer against facts fixed outside itself (CPU only)."""
import pytest

import v2_pins as V


@pytest.mark.parametrize("check", V.V2_CHECKS, ids=lambda f: f.__name__)
def test_v2_pin(check):
    check()
