"""Planted mistakes in copies of the oracle must each fail at least one pin.

Each mutant is the oracle's C source with one plausible mistake (a dropped
term, a wrong sign, a wrong index, a transposed operand) compiled into a
temporary library; the pins of ``oracle_pins`` then run against it.  The real
oracle is never modified.  CPU only.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "drop_eta_in_momentum": ("*m = mu * (*m) - e * kt[i] * vtt[j];",
                             "*m = mu * (*m) - kt[i] * vtt[j];"),
    "sign_of_momentum_write": ("*m = mu * (*m) - e * kt[i] * vtt[j];",
                               "*m = mu * (*m) + e * kt[i] * vtt[j];"),
    "mu_replaced_by_alpha": ("*m = mu * (*m) - e * kt[i] * vtt[j];",
                             "*m = alpha * (*m) - e * kt[i] * vtt[j];"),
    "sign_of_fast_weight_update": ("S[ij] = alpha * S[ij] - b * M[ij];",
                                   "S[ij] = alpha * S[ij] + b * M[ij];"),
    "drop_alpha_decay_of_S": ("S[ij] = alpha * S[ij] - b * M[ij];",
                              "S[ij] = S[ij] - b * M[ij];"),
    "p_without_alpha": ("for (int i = 0; i < dk; ++i) p[i] = alpha * kt[i];",
                        "for (int i = 0; i < dk; ++i) p[i] = kt[i];"),
    "transposed_S_in_vtilde": ("vtt[j] -= S[(ptrdiff_t)i * dv + j] * p[i];",
                               "vtt[j] -= S[(ptrdiff_t)j * dv + i] * p[i];"),
    "transposed_S_in_output": ("ot[j] += S[(ptrdiff_t)i * dv + j] * qhat[i];",
                               "ot[j] += S[(ptrdiff_t)j * dv + i] * qhat[i];"),
    "sign_of_output_correction": ("qhat[i] = qt[i] - d * kt[i];",
                                  "qhat[i] = qt[i] + d * kt[i];"),
    "drop_output_correction": ("qhat[i] = qt[i] - d * kt[i];", "qhat[i] = qt[i];"),
    "mu_not_exponentiated": ("const double mu = exp(mu_log[(ptrdiff_t)t * gate_stride]);",
                             "const double mu = 1.0 + mu_log[(ptrdiff_t)t * gate_stride];"),
    "v_not_subtracted_state": ("for (int j = 0; j < dv; ++j) vtt[j] = vv[j];",
                               "for (int j = 0; j < dv; ++j) vtt[j] = 2.0 * vv[j];"),
    "gamma_drop_eta": ("acc *= eta[gi];", "acc *= 1.0;"),
    "gamma_swapped_mu_ratio": ("exp(lm_c[j] - lm_c[i])", "exp(lm_c[i] - lm_c[j])"),
    "gamma_alpha_ratio_wrong_end": ("exp(la_c[r] - la_c[j])", "exp(la_c[r] - la_c[i])"),
    "lc_drop_beta": ("s += exp(log(beta[g]) + lm_c[j] - la_c[j] - mx);",
                     "s += exp(lm_c[j] - la_c[j] - mx);"),
    "la_off_by_one": ("la_c[r] = sa;\n", "la_c[r] = sa - alpha_log[g];\n"),
    "gamma_strict_lower": ("if (r < L && i <= r) {", "if (r < L && i < r) {"),
    "gates_cos_sin_swapped": ("alpha_log[i] = log(ct * ct) + log_sigmoid(a[i]);",
                              "alpha_log[i] = log(st * st) + log_sigmoid(a[i]);"),
    "gates_theta_without_s": ("const double theta = atan(e * s);", "const double theta = atan(e);"),
    "gates_eta_tanh_without_shift": ("? tanh(x_eta[i]) + 1.0 :", "? tanh(x_eta[i]) :"),
    "gates_clamp_as_upper_bound": ("mu_log[i] = lm > mu_log_min ? lm : mu_log_min;",
                                   "mu_log[i] = lm < mu_log_min ? lm : mu_log_min;"),
    "gates_beta_not_squared": ("beta[i] = st * st * exp(log_sigmoid(b[i]));",
                               "beta[i] = st * exp(log_sigmoid(b[i]));"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation anchor for {name} not unique/present"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    lib = oracle.load(oracle.compile_oracle(str(src), str(tmp_path / f"lib{name}.so")))
    failures = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError as e:  # a pin caught the planted mistake
            failures.append(f"{pin.__name__}: {str(e)[:80]}")
    assert failures, f"no pin catches mutant {name}"
