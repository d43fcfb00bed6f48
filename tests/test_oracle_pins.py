"""The fp64 oracle against its pins (hand-worked values, closed form, special
cases, spectrum, chunkwise restatement).  CPU only."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(oracle.load())


def test_reordering_identity_bruteforce():
    """sum_{i<=t} sum_{j<=i} a_i b_j == sum_{i<=t} sum_{j=i}^{t} a_j b_i (row scan vs
    column scan of the lower triangle), by brute force on tiny t."""
    import numpy as np
    rng = np.random.default_rng(5)
    for t in range(1, 17):
        a, b = rng.standard_normal(t), rng.standard_normal(t)
        rows = sum(a[i] * b[j] for i in range(t) for j in range(i + 1))
        cols = sum(a[j] * b[i] for i in range(t) for j in range(i, t))
        assert abs(rows - cols) <= 1e-12 * max(1.0, abs(rows))
