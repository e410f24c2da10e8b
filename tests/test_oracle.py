"""The CPU oracle against its pins (no GPU needed)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle)


def test_oracle_uses_threads():
    import numpy as np
    q = np.random.default_rng(0).standard_normal((2, 4, 8, 4))
    oracle.attn_fwd(q, q, q)
    assert oracle.threads_used() >= 1
