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


@pytest.mark.parametrize("T,C", [(7, 3), (13, 4), (21, 8), (9, 64)])
def test_chunk_backward_restatement(T, C):
    """The chunkwise backward algebra (the reverse chain of state adjoints plus
    per-chunk gradients through the coefficient adjoints) equals the gradient
    oracle, with some eta and beta exactly zero (structural masks, not value
    masks) and a ragged last chunk."""
    import numpy as np
    from chunk_reference import chunk_backward
    from oracle import backward as ob
    from oracle_pins import _rand_case
    rng = np.random.default_rng(T * 100 + C)
    B, H, d = 1, 2, 4
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    et[0, T // 3, 0] = 0.0
    be[0, T // 2, 1] = 0.0
    do = rng.standard_normal((B, T, H, d))
    dS = rng.standard_normal((B, H, d, d))
    dM = rng.standard_normal((B, H, d, d))
    ref = ob.chunk_bwd(q, k, v, al, ml, be, et, 0.5, S0, M0, do, dS, dM)
    got = chunk_backward(q, k, v, al, ml, be, et, 0.5, S0, M0, do, dS, dM, C=C)
    for name in ref:
        err = np.max(np.abs(got[name] - ref[name])) / max(1.0, np.max(np.abs(ref[name])))
        assert err < 1e-12, (name, err)
