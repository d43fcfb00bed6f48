"""Pins of the fp64 oracle to results fixed by the pages or by mathematics.

Each ``pin_*`` function takes an oracle library handle (``oracle.load(path)``)
and raises AssertionError when the oracle disagrees.  ``test_oracle_pins``
runs them on the real oracle; ``test_oracle_mutants`` runs them on copies of
the oracle with planted mistakes and checks that some pin fails each time.

Sources ("MDN: Parallelizing Stepwise Momentum for Delta Linear Attention"):
  recurrence ............ paper.rainbus.top summary, step 1; ijyty.com, section 3
  unrolled closed form .. summary, step 2 (eta_i on write i: a reading)
  row<->column reordering summary, step 3; ijyty.com, section 4
  chunkwise form ........ summary, step 4
  spectrum lambda+- ..... summary, step 6; novelty paragraph; ijyty.com, section 5
  mu = 0 ablation ....... ijyty.com, section 8 (reduces to a gated delta rule)
  gate parameterisation . summary, step 6; ijyty.com, sections 5 and 8
  ||Delta S_t||_F ........ ijyty.com, section 8 (decoding diagnostic)
  packed sequences ...... the pages' one-sequence recurrence per sequence (their
                          silence on packing read as independence)
  gradients ............. summary, step 7; ijyty.com, section 6 (training saves
                          vtilde, rebuilds S and M in the backward pass)
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np

import oracle
from chunk_reference import chunk_forward

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _frac(x) -> float:
    return float(Fraction(x))


def _rand_case(rng, B, T, H, d, state=True, alpha_lo=0.3, alpha_hi=0.95,
               mu_lo=0.4, mu_hi=0.95):
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, d))
    al = np.log(rng.uniform(alpha_lo, alpha_hi, (B, T, H)))
    ml = np.log(rng.uniform(mu_lo, mu_hi, (B, T, H)))
    be = rng.uniform(0.05, 0.6, (B, T, H))
    et = rng.uniform(0.2, 1.8, (B, T, H))
    S0 = rng.standard_normal((B, H, d, d)) * 0.3 if state else None
    M0 = rng.standard_normal((B, H, d, d)) * 0.3 if state else None
    return q, k, v, al, ml, be, et, S0, M0


def _close(a, b, tol, what):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b)))
    assert err <= tol, f"{what}: max err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- hand-worked
def _golden_case(lib, name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)
    T, d = len(g["q"]), len(g["q"][0])
    shp = (1, T, 1, d)
    q = np.array(g["q"], dtype=np.float64).reshape(shp)
    k = np.array(g["k"], dtype=np.float64).reshape(shp)
    v = np.array(g["v"], dtype=np.float64).reshape(shp)
    gate = lambda key: np.array(g[key], dtype=np.float64).reshape(1, T, 1)
    al, ml = np.log(gate("alpha")), np.log(gate("mu"))
    S0 = None
    if "S0" in g:
        S0 = np.array([[_frac(x) for x in row] for row in g["S0"]]).reshape(1, 1, d, d)
    o, vt, S_T, M_T = oracle.chunk_fwd(q, k, v, al, ml, gate("beta"), gate("eta"),
                                       g["d"], S0, None, lib=lib)
    exp = g["expected"]
    conv = lambda m: np.array([[_frac(x) for x in row] for row in m])
    _close(vt.reshape(T, d), conv(exp["vtilde"]), 1e-14, f"{name} vtilde")
    _close(o.reshape(T, d), conv(exp["o"]), 1e-14, f"{name} o")
    _close(S_T.reshape(d, d), conv(exp["S_T"]), 1e-14, f"{name} S_T")
    _close(M_T.reshape(d, d), conv(exp["M_T"]), 1e-14, f"{name} M_T")


def pin_hand_scalar(lib):
    _golden_case(lib, "hand_scalar_d1_T3.json")


def pin_hand_matrix(lib):
    _golden_case(lib, "hand_matrix_d2_T2.json")


# ---------------------------------------------------------------- closed form
def pin_closed_form(lib):
    """Unrolled form (summary step 2, with eta_i on write i) at every prefix t."""
    rng = np.random.default_rng(11)
    T, d = 24, 5
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, 1, T, 1, d)
    dcorr = 0.5
    _, vt, _, _ = oracle.chunk_fwd(q, k, v, al, ml, be, et, dcorr, S0, M0, lib=lib)
    a, m, b_, e = al[0, :, 0], ml[0, :, 0], be[0, :, 0], et[0, :, 0]
    K, V, Vt, Q = k[0, :, 0], v[0, :, 0], vt[0, :, 0], q[0, :, 0]
    abar, mbar = np.exp(np.cumsum(a)), np.exp(np.cumsum(m))
    c = np.cumsum(b_ * mbar / abar)
    for t in range(1, T + 1):
        # M_t = mubar_t M0 - sum_i (mubar_t/mubar_i) eta_i k_i vt_i^T
        Mt = mbar[t - 1] * M0[0, 0].copy()
        St = abar[t - 1] * S0[0, 0] - abar[t - 1] * c[t - 1] * M0[0, 0]
        for i in range(1, t + 1):
            outer = np.outer(K[i - 1], Vt[i - 1])
            Mt -= (mbar[t - 1] / mbar[i - 1]) * e[i - 1] * outer
            c_im1 = c[i - 2] if i >= 2 else 0.0
            gam = abar[t - 1] / mbar[i - 1] * (c[t - 1] - c_im1)
            St += gam * e[i - 1] * outer
        o_t, _, S_t, M_t = oracle.chunk_fwd(q[:, :t], k[:, :t], v[:, :t], al[:, :t],
                                            ml[:, :t], be[:, :t], et[:, :t], dcorr,
                                            S0, M0, lib=lib)
        _close(S_t[0, 0], St, 1e-11, f"closed-form S_{t}")
        _close(M_t[0, 0], Mt, 1e-11, f"closed-form M_{t}")
        qh = Q[t - 1] - dcorr * K[t - 1]
        _close(o_t[0, t - 1, 0], St.T @ qh, 1e-11, f"closed-form o_{t}")
    # vtilde against its definition using the closed-form S_{t-1}
    S_prev = S0[0, 0].copy()
    for t in range(1, T + 1):
        _close(Vt[t - 1], V[t - 1] - np.exp(a[t - 1]) * S_prev.T @ K[t - 1], 1e-11,
               f"vtilde_{t}")
        _, _, S_pt, _ = oracle.chunk_fwd(q[:, :t], k[:, :t], v[:, :t], al[:, :t],
                                         ml[:, :t], be[:, :t], et[:, :t], dcorr,
                                         S0, M0, lib=lib)
        S_prev = S_pt[0, 0]


# ---------------------------------------------------------------- mu = 0
def pin_mu_zero_gated_delta_rule(lib):
    """mu = 0: S_t = alpha_t (I - beta_t eta_t k_t k_t^T) S_{t-1} + beta_t eta_t k_t v_t^T."""
    rng = np.random.default_rng(12)
    T, d = 20, 6
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, 1, T, 1, d)
    ml[:] = -np.inf
    dcorr = 0.25
    o, vt, S_T, M_T = oracle.chunk_fwd(q, k, v, al, ml, be, et, dcorr, S0, M0, lib=lib)
    S = S0[0, 0].copy()
    for t in range(T):
        kt, vv = k[0, t, 0], v[0, t, 0]
        w = be[0, t, 0] * et[0, t, 0]
        S = np.exp(al[0, t, 0]) * (np.eye(d) - w * np.outer(kt, kt)) @ S + w * np.outer(kt, vv)
        _close(o[0, t, 0], S.T @ (q[0, t, 0] - dcorr * kt), 1e-12, f"GDN o_{t}")
    _close(S_T[0, 0], S, 1e-12, "GDN S_T")


# ---------------------------------------------------------------- spectrum
def _one_step_matrix(lib, dk, dv, alpha, mu, beta, eta, kvec):
    n = dk * dv
    A = np.zeros((2 * n, 2 * n))
    zero = np.zeros((1, 1, dk))
    g = lambda x: np.array([[x]], dtype=np.float64)
    for col in range(2 * n):
        e = np.zeros(2 * n)
        e[col] = 1.0
        S = e[:n].reshape(1, 1, dk, dv)
        M = e[n:].reshape(1, 1, dk, dv)
        _, _, S1, M1 = oracle.step(zero, kvec.reshape(1, 1, dk), np.zeros((1, 1, dv)),
                                   g(np.log(alpha)), g(np.log(mu)), g(beta), g(eta), 0.0,
                                   S, M, lib=lib)
        A[:, col] = np.concatenate([S1.ravel(), M1.ravel()])
    return A


def _match_multiset(got, want, tol):
    got = list(got)
    for w in want:
        j = int(np.argmin([abs(g - w) for g in got]))
        assert abs(got[j] - w) <= tol, f"eigenvalue {w} not found (closest {got[j]})"
        got.pop(j)


def pin_spectrum(lib):
    """Block transition [S;M]_t = A_t [S;M]_{t-1} at d=2 (and d_k=3, d_v=2 via dk=dv=3):
    spectrum {alpha x (d_k-1)d_v, mu x (d_k-1)d_v, lambda+- x d_v each} with
    lambda+- = (tau +- sqrt(tau^2 - 4 alpha mu)) / 2, tau = alpha + mu - alpha beta eta |k|^2."""
    cases = [  # (alpha, mu, beta, eta, k): complex pair, real pair, |k| != 1
        (0.7, 0.6, 0.3, 0.9, np.array([0.6, 0.8])),
        (0.2, 0.9, 0.7, 1.9, np.array([1.0, 0.0])),
        (0.5, 0.5, 0.25, 1.0, np.array([0.9, -0.7])),
        (0.6, 0.45, 0.35, 1.3, np.array([0.3, -0.5, 0.8])),
    ]
    for alpha, mu, beta, eta, kv in cases:
        dk = dv = kv.size
        A = _one_step_matrix(lib, dk, dv, alpha, mu, beta, eta, kv)
        kappa = float(kv @ kv)
        tau = alpha + mu - alpha * beta * eta * kappa
        disc = complex(tau * tau - 4 * alpha * mu)
        lp, lm_ = (tau + disc ** 0.5) / 2, (tau - disc ** 0.5) / 2
        want = ([alpha] * ((dk - 1) * dv) + [mu] * ((dk - 1) * dv)
                + [lp] * dv + [lm_] * dv)
        _match_multiset(np.linalg.eigvals(A), want, 1e-7)


# ---------------------------------------------------------------- chunk form
def pin_chunked_form(lib):
    """The chunkwise restatement equals the stepwise oracle for every chunk length,
    ragged tails included, with non-zero entering states."""
    rng = np.random.default_rng(13)
    B, T, H, d = 2, 37, 2, 4
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    ref = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0, lib=lib)
    for C in (1, 2, 4, 16, 64):
        got = chunk_forward(q, k, v, al, ml, be, et, 0.5, S0, M0, C=C)
        for name, x, y in zip(("o", "vtilde", "S_T", "M_T"), got, ref):
            _close(x, y, 1e-10, f"chunked C={C} {name}")


# ---------------------------------------------------------------- coefficients
def pin_chunk_coeffs(lib):
    """Per-chunk la, lm, lc, Gamma reproduce the chunk-end state through the unrolled
    form; Gamma's diagonal is beta_r eta_r and Gamma obeys
    Gamma_{r,i} = alpha_r Gamma_{r-1,i} + eta_i beta_r mubar_r / mubar_i."""
    rng = np.random.default_rng(14)
    B, T, H, d, C = 1, 45, 2, 3, 16
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    la, lm, lc, G = oracle.chunk_coeffs(al, ml, be, et, C, lib=lib)
    _, vt, _, _ = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0, lib=lib)
    NT = (T + C - 1) // C
    for h in range(H):
        S, M = S0[0, h].copy(), M0[0, h].copy()
        for n in range(NT):
            t0, t1 = n * C, min(T, n * C + C)
            L = t1 - t0
            Gn = G[0, h, n]
            a_c, m_c, c_c = la[0, h, t0:t1], lm[0, h, t0:t1], lc[0, h, t0:t1]
            # log-domain quantities against cumulative products of the gates
            assert np.allclose(np.exp(a_c), np.cumprod(np.exp(al[0, t0:t1, h])), rtol=1e-12)
            assert np.allclose(np.exp(m_c), np.cumprod(np.exp(ml[0, t0:t1, h])), rtol=1e-12)
            terms = be[0, t0:t1, h] * np.exp(m_c) / np.exp(a_c)
            assert np.allclose(np.exp(c_c), np.cumsum(terms), rtol=1e-12)
            alpha = np.exp(al[0, t0:t1, h])
            for r in range(L):
                assert abs(Gn[r, r] - be[0, t0 + r, h] * et[0, t0 + r, h]) < 1e-13
                for i in range(r):
                    want = (alpha[r] * Gn[r - 1, i]
                            + et[0, t0 + i, h] * be[0, t0 + r, h] * np.exp(m_c[r] - m_c[i]))
                    assert abs(Gn[r, i] - want) <= 1e-12 * max(1.0, abs(want))
            assert np.all(np.triu(Gn, 1) == 0)
            assert np.all(Gn[L:, :] == 0) and np.all(Gn[:, L:] == 0)
            K, Vt = k[0, t0:t1, h], vt[0, t0:t1, h]
            abarL, bL = np.exp(a_c[-1]), np.exp(a_c[-1] + c_c[-1])
            w_m = et[0, t0:t1, h] * np.exp(m_c[-1] - m_c)
            S_new = abarL * S - bL * M + K.T @ (Gn[L - 1, :L][:, None] * Vt)
            M_new = np.exp(m_c[-1]) * M - K.T @ (w_m[:, None] * Vt)
            S, M = S_new, M_new
        _, _, S_T, M_T = oracle.chunk_fwd(q[:, :, h:h + 1], k[:, :, h:h + 1],
                                          v[:, :, h:h + 1], al[:, :, h:h + 1],
                                          ml[:, :, h:h + 1], be[:, :, h:h + 1],
                                          et[:, :, h:h + 1], 0.5, S0[:, h:h + 1],
                                          M0[:, h:h + 1], lib=lib)
        _close(S, S_T[0, 0], 1e-11, f"coeffs S_T head {h}")
        _close(M, M_T[0, 0], 1e-11, f"coeffs M_T head {h}")


# ---------------------------------------------------------------- decode step
def pin_step_matches_sequence(lib):
    """T calls of the one-token step equal one pass over the T tokens (the pages'
    claim that stepwise decoding behaves exactly as chunkwise training)."""
    rng = np.random.default_rng(15)
    B, T, H, d = 2, 9, 3, 4
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    o_ref, vt_ref, S_ref, M_ref = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0,
                                                   lib=lib)
    S, M = S0, M0
    for t in range(T):
        o, vt, S, M = oracle.step(q[:, t], k[:, t], v[:, t], al[:, t], ml[:, t], be[:, t],
                                  et[:, t], 0.5, S, M, lib=lib)
        _close(o, o_ref[:, t], 1e-13, f"step o_{t}")
        _close(vt, vt_ref[:, t], 1e-13, f"step vtilde_{t}")
    _close(S, S_ref, 1e-13, "step S_T")
    _close(M, M_ref, 1e-13, "step M_T")


def pin_resume(lib):
    """Running [0, T1) then [T1, T) with the first call's S_T, M_T as the second's
    S0, M0 equals one call over [0, T)."""
    rng = np.random.default_rng(16)
    B, T, H, d = 1, 30, 2, 4
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    ref = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0, lib=lib)
    T1 = 13
    a = oracle.chunk_fwd(q[:, :T1], k[:, :T1], v[:, :T1], al[:, :T1], ml[:, :T1],
                         be[:, :T1], et[:, :T1], 0.5, S0, M0, lib=lib)
    b = oracle.chunk_fwd(q[:, T1:], k[:, T1:], v[:, T1:], al[:, T1:], ml[:, T1:],
                         be[:, T1:], et[:, T1:], 0.5, a[2], a[3], lib=lib)
    _close(np.concatenate([a[0], b[0]], axis=1), ref[0], 1e-13, "resume o")
    _close(b[2], ref[2], 1e-13, "resume S_T")



def pin_varlen(lib):
    """Sequences packed along the token axis: (1) N sequences of one length equal
    the batched pass with B = N; (2) lengths 0, 1, 5, 13 equal the one-token
    step run over the packed rows with the state reset to S0[s] at every
    sequence start; (3) an empty sequence returns its S0, M0."""
    rng = np.random.default_rng(17)
    N, L, H, d = 3, 7, 2, 4
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, N, L, H, d)
    flat = lambda x: x.reshape((N * L,) + x.shape[2:])
    cu = np.arange(N + 1) * L
    ref = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0, lib=lib)
    got = oracle.chunk_fwd_varlen(flat(q), flat(k), flat(v), flat(al), flat(ml), flat(be),
                                  flat(et), cu, 0.5, S0, M0, lib=lib)
    for name, g, r in zip(("o", "vtilde"), got[:2], ref[:2]):
        assert np.array_equal(g, flat(r)), f"varlen equal-length {name}"
    assert np.array_equal(got[2], ref[2]) and np.array_equal(got[3], ref[3])

    lens = [0, 5, 1, 13, 0]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt, N = int(cu[-1]), len(lens)
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, 1, Tt, H, d)
    q, k, v, al, ml, be, et = (x[0] for x in (q, k, v, al, ml, be, et))
    S0 = rng.standard_normal((N, H, d, d))
    M0 = rng.standard_normal((N, H, d, d))
    o, vt, S_T, M_T = oracle.chunk_fwd_varlen(q, k, v, al, ml, be, et, cu, 0.5, S0, M0, lib=lib)
    for s in range(N):
        S, M = S0[s:s + 1], M0[s:s + 1]
        for t in range(cu[s], cu[s + 1]):
            to, tvt, S, M = oracle.step(q[t][None], k[t][None], v[t][None], al[t][None],
                                        ml[t][None], be[t][None], et[t][None], 0.5, S, M,
                                        lib=lib)
            _close(o[t], to[0], 1e-13, f"varlen o seq {s} token {t}")
            _close(vt[t], tvt[0], 1e-13, f"varlen vtilde seq {s} token {t}")
        _close(S_T[s], S[0], 1e-13, f"varlen S_T seq {s}")
        _close(M_T[s], M[0], 1e-13, f"varlen M_T seq {s}")
        if lens[s] == 0:
            assert np.array_equal(S_T[s], S0[s]) and np.array_equal(M_T[s], M0[s])


# ---------------------------------------------------------------- backward
def pin_backward_forward_is_the_oracle(lib):
    """The torch recurrence that the gradient oracle differentiates equals the
    C oracle's forward pass (o, vtilde, S_T, M_T)."""
    from oracle import backward as ob
    import torch
    rng = np.random.default_rng(31)
    B, T, H, d = 2, 11, 2, 5
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    ref = oracle.chunk_fwd(q, k, v, al, ml, be, et, 0.5, S0, M0, lib=lib)
    tt = lambda x: torch.as_tensor(x, dtype=torch.float64)
    got = ob.forward(*(tt(x) for x in (q, k, v, al, ml, be, et)), 0.5, tt(S0), tt(M0))
    for name, g, r in zip(("o", "vtilde", "S_T", "M_T"), got, ref):
        _close(g.numpy(), r, 1e-12, f"torch forward {name}")


def pin_backward_finite_differences(lib):
    """Every gradient entry against a central difference of the loss
    (h = 1e-6, fp64) on a case with non-zero entering states and all three
    cotangents."""
    from oracle import backward as ob
    rng = np.random.default_rng(32)
    B, T, H, d = 1, 6, 2, 3
    q, k, v, al, ml, be, et, S0, M0 = _rand_case(rng, B, T, H, d)
    do = rng.standard_normal((B, T, H, d))
    dS = rng.standard_normal((B, H, d, d))
    dM = rng.standard_normal((B, H, d, d))
    args = dict(q=q, k=k, v=v, alpha_log=al, mu_log=ml, beta=be, eta=et)
    g = ob.chunk_bwd(q, k, v, al, ml, be, et, 0.5, S0, M0, do, dS, dM)
    states = dict(S0=S0, M0=M0)
    h = 1e-6
    for name in list(args) + list(states):
        base = args if name in args else states
        x = base[name]
        grad = g["d" + name]
        assert grad.shape == x.shape, name
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            lp = ob.loss_value(**{**args, **states, name: xp}, d=0.5, do=do, dS_T=dS, dM_T=dM)
            lm = ob.loss_value(**{**args, **states, name: xm}, d=0.5, do=do, dS_T=dS, dM_T=dM)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def pin_backward_single_token(lib):
    """One token from zero states: S_1 = beta eta k v^T and o = beta eta (k.qhat) v,
    so with L = <do, o> + <dS, S_1>: dv = beta eta ((k.qhat) do + dS^T k),
    dq = beta eta (v.do) k, dk = beta eta ((v.do)(qhat - d k) + dS v),
    dbeta = eta X, deta = beta X with X = (k.qhat)(v.do) + k^T dS v, and no
    dependence on alpha or mu (the states they scale are zero)."""
    from oracle import backward as ob
    rng = np.random.default_rng(33)
    d, dc = 4, 0.5
    q, k, v, do = (rng.standard_normal((1, 1, 1, d)) for _ in range(4))
    dS = rng.standard_normal((1, 1, d, d))
    al, ml = np.full((1, 1, 1), -0.3), np.full((1, 1, 1), -0.7)
    be, et = np.full((1, 1, 1), 0.6), np.full((1, 1, 1), 1.3)
    g = ob.chunk_bwd(q, k, v, al, ml, be, et, dc, None, None, do, dS, None)
    kk, vv, qq, oo, SS = k[0, 0, 0], v[0, 0, 0], q[0, 0, 0], do[0, 0, 0], dS[0, 0]
    qh = qq - dc * kk
    c, w = 0.6 * 1.3, (kk @ qh) * (vv @ oo) + kk @ SS @ vv
    _close(g["dv"][0, 0, 0], c * ((kk @ qh) * oo + SS.T @ kk), 1e-13, "1-token dv")
    _close(g["dq"][0, 0, 0], c * (vv @ oo) * kk, 1e-13, "1-token dq")
    _close(g["dk"][0, 0, 0], c * ((vv @ oo) * (qh - dc * kk) + SS @ vv), 1e-13, "1-token dk")
    _close(g["dbeta"][0, 0, 0], 1.3 * w, 1e-13, "1-token dbeta")
    _close(g["deta"][0, 0, 0], 0.6 * w, 1e-13, "1-token deta")
    _close(g["dalpha_log"], np.zeros((1, 1, 1)), 1e-15, "1-token dalpha")
    _close(g["dmu_log"], np.zeros((1, 1, 1)), 1e-15, "1-token dmu")

# ---------------------------------------------------------------- gates
def _logsig(x):
    return -np.logaddexp(0.0, -np.asarray(x, dtype=np.float64))


def pin_gates_special_points(lib):
    """theta = arctan(eta s): s = 0 gives theta = 0 (alpha = sigmoid(a), beta = 0);
    x = 0 gives eta = 1 for both activations, so s = 1 gives theta = pi/4
    (cos^2 = sin^2 = 1/2).  mu_log is log sigmoid(c) above the clamp, the clamp
    below it."""
    a = np.array([-3.0, 0.0, 2.5]); b = np.array([1.0, -0.5, 0.0]); c = np.array([0.0, -5.0, 4.0])
    x0 = np.zeros(3)
    for act in ("tanh", "2sigmoid"):
        al, ml, be, et = oracle.gates(np.array([0.3, -1.2, 2.0]), a, b, c, s=0.0,
                                      mu_log_min=-1.0, eta_act=act, lib=lib)
        _close(al, _logsig(a), 1e-15, f"{act} s=0 alpha_log")
        _close(be, np.zeros(3), 1e-15, f"{act} s=0 beta")
        al, ml, be, et = oracle.gates(x0, a, b, c, s=1.0, mu_log_min=-1.0, eta_act=act, lib=lib)
        _close(et, np.ones(3), 1e-15, f"{act} eta(0)")
        _close(al, np.log(0.5) + _logsig(a), 1e-14, f"{act} theta=pi/4 alpha_log")
        _close(be, 0.5 / (1.0 + np.exp(-b)), 1e-14, f"{act} theta=pi/4 beta")
        # log sigmoid(0) = -log 2 > -1; log sigmoid(-5) < -1 clamps; log sigmoid(4) ~ -0.018
        _close(ml, [-np.log(2.0), -1.0, -np.log1p(np.exp(-4.0))], 1e-15, f"{act} mu_log")


def pin_gates_identities(lib):
    """On random pre-activations: alpha/sigmoid(a) + beta/sigmoid(b) = 1
    (cos^2 + sin^2); cos^2(arctan u) = 1/(1+u^2) with u = eta s; and the two
    eta activations agree through tanh(x) + 1 = 2 sigmoid(2x)."""
    rng = np.random.default_rng(21)
    n = 257
    x, a, b, c = (rng.standard_normal(n) * 2.0 for _ in range(4))
    s = 1.7
    al, ml, be, et = oracle.gates(x, a, b, c, s=s, mu_log_min=-2.0, eta_act="tanh", lib=lib)
    sa, sb = 1.0 / (1.0 + np.exp(-a)), 1.0 / (1.0 + np.exp(-b))
    _close(np.exp(al) / sa + be / sb, np.ones(n), 1e-13, "cos^2 + sin^2")
    _close(al, -np.log1p((et * s) ** 2) + _logsig(a), 1e-13, "cos^2(arctan u)")
    assert np.all(et > 0.0) and np.all(et < 2.0), "eta in (0, 2)"
    assert np.all(ml >= -2.0) and np.all(ml < 0.0), "mu_log in [clamp, 0)"
    al2, ml2, be2, et2 = oracle.gates(2.0 * x, a, b, c, s=s, mu_log_min=-2.0,
                                      eta_act="2sigmoid", lib=lib)
    _close(et2, et, 1e-14, "tanh(x)+1 = 2 sigmoid(2x)")
    _close(al2, al, 1e-13, "same alpha through either activation")
    _close(be2, be, 1e-13, "same beta through either activation")


def pin_step_delta_norm(lib):
    """||S_t - S_{t-1}||_F of one decode step: from zero states the first write is
    S_1 = beta eta k v^T, so the norm is beta eta ||k|| ||v||; with alpha = 1 and
    beta = 0 the fast weight does not move."""
    rng = np.random.default_rng(23)
    B, H, d = 2, 3, 5
    q, k, v = (rng.standard_normal((B, H, d)) for _ in range(3))
    be, et = rng.uniform(0.1, 0.9, (B, H)), rng.uniform(0.2, 1.8, (B, H))
    al, ml = np.log(rng.uniform(0.3, 0.9, (B, H))), np.log(rng.uniform(0.4, 0.9, (B, H)))
    Z = np.zeros((B, H, d, d))
    _, _, S1, _ = oracle.step(q, k, v, al, ml, be, et, 0.5, Z, Z, lib=lib)
    want = be * et * np.linalg.norm(k, axis=-1) * np.linalg.norm(v, axis=-1)
    _close(oracle.step_delta_norm(Z, S1), want, 1e-13, "first write norm")
    S0, M0 = rng.standard_normal((B, H, d, d)), rng.standard_normal((B, H, d, d))
    _, _, S2, _ = oracle.step(q, k, v, np.zeros((B, H)), ml, np.zeros((B, H)), et, 0.5, S0, M0,
                              lib=lib)
    _close(oracle.step_delta_norm(S0, S2), np.zeros((B, H)), 1e-15, "alpha=1, beta=0")


ALL_PINS = [pin_hand_scalar, pin_hand_matrix, pin_closed_form, pin_mu_zero_gated_delta_rule,
            pin_spectrum, pin_chunked_form, pin_chunk_coeffs, pin_step_matches_sequence,
            pin_resume, pin_varlen, pin_gates_special_points, pin_gates_identities,
            pin_step_delta_norm, pin_backward_forward_is_the_oracle,
            pin_backward_finite_differences, pin_backward_single_token]
