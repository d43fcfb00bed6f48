"""K-1 (chunk coefficients) on the GPU against the oracle's plain definitions."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from parity import to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,T", [(0, 256), (1, 300), (3, 1000)])
def test_gate_prep_matches_oracle(cfg, T):
    spec = mi.replace(mi.WORKLOADS[cfg], B=2, H=3, T=T)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    la, lm, lc, bco, gam = mdn.chunk_gate_prep(dev["alpha_log"], dev["mu_log"], dev["beta"],
                                               dev["eta"])
    torch.cuda.synchronize()
    ola, olm, olc, og = oracle.chunk_coeffs(inp.alpha_log, inp.mu_log, inp.beta, inp.eta, 64)
    la, lm, lc, bco, gam = (to_np(x) for x in (la, lm, lc, bco, gam))
    C, NT = 64, (T + 63) // 64
    # log-domain sums: absolute error relative to the magnitude of the sum
    for got, ref in ((la, ola), (lm, olm), (lc, olc)):
        g = got[:, :, :T]
        assert np.all(np.isfinite(g))
        assert np.max(np.abs(g - ref) / (1.0 + np.abs(ref))) < 2e-5
    b_ref = np.exp(ola + olc)
    assert np.max(np.abs(bco[:, :, :T] - b_ref) / (1e-30 + np.abs(b_ref))) < 5e-4
    # Gamma: per row, error relative to the row's largest entry
    for bb in range(2):
        for h in range(3):
            for n in range(NT):
                L = min(C, T - n * C)
                G, R = gam[bb, h, n], og[bb, h, n]
                err = np.abs(G[:L, :L] - R[:L, :L]).max(axis=1) / np.abs(R[:L, :L]).max(axis=1)
                assert err.max() < 2e-5, (bb, h, n, err.max())
                assert np.all(np.triu(G, 1) == 0)
                # padded rows repeat the last real row (steps that change nothing)
                if L < C:
                    assert np.allclose(G[L:, :], G[L - 1:L, :])
                    assert np.all(G[:, L:] == 0)


def test_gate_prep_stress_regime():
    """alpha -> 1 with mu at its clamp e^-1: c_r - c_{i-1} cancels in the
    log-broadcast form; the column recurrence keeps Gamma accurate."""
    spec = mi.replace(mi.WORKLOADS[1], B=1, H=4, T=256, a_mean=6.0, x_mean=-1.5, c_mean=-5.0)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    *_, gam = mdn.chunk_gate_prep(dev["alpha_log"], dev["mu_log"], dev["beta"], dev["eta"])
    *_, og = oracle.chunk_coeffs(inp.alpha_log, inp.mu_log, inp.beta, inp.eta, 64)
    gam = to_np(gam)
    err = np.abs(gam - og).max() / np.abs(og).max()
    assert err < 1e-5
