"""The oracle's backbone stack against facts fixed outside itself (CPU only)."""
import pytest

import stack_pins as S


@pytest.mark.parametrize("check", S.STACK_CHECKS, ids=lambda f: f.__name__)
def test_stack_pin(check):
    check()
