"""The seeded input generator: storage rounding and the gate constraints the
pages require of stable gates.  CPU only."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 3.0e-3, -7.77e5],
                 dtype=np.float32)
    bits = mi.bf16_round_bits(x)
    assert bits[0] == 0x3F80 and bits[1] == 0x3F80 and bits[2] == 0x3F82
    assert bits[3] == 0xBF80
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(bits, ref)
    rng = np.random.default_rng(0)
    y = rng.standard_normal(100000).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(mi.bf16_round_bits(y), ref)
    assert np.array_equal(mi.bf16_bits_to_f32(ref), torch.from_numpy(y).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("cfg", range(len(mi.WORKLOADS)))
def test_gates_satisfy_stability_constraints(cfg):
    """Stability inequality -(1-a)(1-mu) <= a beta eta |k|^2 <= (1+a)(1+mu) (novelty
    paragraph of the paper.rainbus.top summary) and non-negative real parts of
    lambda+- (summary step 6), on the generated gates and stored keys."""
    spec = mi.WORKLOADS[cfg]
    spec = mi.replace(spec, B=min(spec.B, 2), T=min(spec.T, 512))
    inp = mi.make_inputs(spec)
    a = np.exp(inp.alpha_log.astype(np.float64))
    mu = np.exp(inp.mu_log.astype(np.float64))
    be, et = inp.beta.astype(np.float64), inp.eta.astype(np.float64)
    kappa = np.sum(inp.k.astype(np.float64) ** 2, axis=-1)
    x = a * be * et * kappa
    assert np.all(-(1 - a) * (1 - mu) <= x) and np.all(x <= (1 + a) * (1 + mu))
    tau = a + mu - x
    assert np.all(tau >= 0)          # Re(lambda+-) = tau/2 or both real roots >= 0
    assert np.all(be <= 1 - a + 1e-6)  # beta <= 1 - alpha
    assert np.all(inp.mu_log >= spec.mu_log_min - 1e-6)
    assert np.all((et > 0) & (et < 2))


def test_generator_is_deterministic():
    s = mi.replace(mi.WORKLOADS[2], B=1, T=128, H=2)
    a, b = mi.make_inputs(s), mi.make_inputs(s)
    for f in ("q_store", "k_store", "v_store", "alpha_log", "mu_log", "beta", "eta", "S0", "M0"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    assert a.S0.std() == pytest.approx(0.01, rel=0.05)
