"""CPU checks that the kernels' rewrites of the pages' definitions are exact.

Each test emulates, in fp64 and in the order the kernel performs them, the
steps of one of the chunk kernels' algorithms, and compares the result with
the oracle or with a library routine.  They test the algorithms (their
algebra and their schedules), not the CUDA code: the GPU parity tests cover
the kernels themselves.

"MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
paper.rainbus.top summary, steps 3-5 and 7 (the chunk form, Gamma,
T = (I + P K^T o Gamma-)^-1, q-hat), and the backward pass the pages train with
(summary step 7; ijyty.com article section 6).
"""
import numpy as np

import mdn_inputs as mi
import oracle

C = 64


def _chunk_gates(seed=7):
    """One chunk of the seeded generator's gates (fp64), as a kernel reads them."""
    inp = mi.make_inputs(mi.Spec("algebra", B=1, T=3 * C, H=2, d=64, dtype="f32", seed=seed))
    sl = (0, slice(C, 2 * C), 1)  # batch 0, chunk 1, head 1
    return tuple(np.asarray(g, dtype=np.float64)[sl] for g in
                 (inp.alpha_log, inp.mu_log, inp.beta, inp.eta)), inp


def _oracle_gamma(inp):
    _, _, _, gamma = oracle.chunk_coeffs(inp.alpha_log, inp.mu_log, inp.beta, inp.eta, C)
    return gamma[0, 1, 1]  # batch 0, head 1, chunk 1


def test_gamma_column_walk_zero_started_matches_oracle():
    """The gate-prep kernel's walk down column i: f_r = mu_r f_{r-1} + [r = i]
    from f = 0, h_r = alpha_r h_{r-1} + beta_r f_r, Gamma_{r,i} = eta_i h_r."""
    (al, ml, be, et), inp = _chunk_gates()
    a, m = np.exp(al), np.exp(ml)
    G = np.zeros((C, C))
    for i in range(C):
        f = h = 0.0
        for r in range(C):
            f = m[r] * f + (1.0 if r == i else 0.0)
            h = a[r] * h + be[r] * f
            G[r, i] = et[i] * h
    ref = _oracle_gamma(inp)
    assert np.abs(G - ref).max() <= 1e-12 * np.abs(ref).max()


def test_gamma_column_walk_predicated_matches_oracle():
    """The intra-chunk kernel's column pass: f = 1 on and above the diagonal and
    f mu_r below it, Gamma = alpha_r Gamma_{r-1} + eta_i beta_r f on and below it."""
    (al, ml, be, et), inp = _chunk_gates(seed=8)
    a, m = np.exp(al), np.exp(ml)
    G = np.zeros((C, C))
    for i in range(C):
        g, f = 0.0, 1.0
        for r in range(C):
            f = f * m[r] if r > i else 1.0
            g = a[r] * g + et[i] * be[r] * f if r >= i else 0.0
            G[r, i] = g
    ref = _oracle_gamma(inp)
    assert np.abs(G - ref).max() <= 1e-12 * np.abs(ref).max()


def _blocked_inverse(A):
    """T = (I + A)^-1 for strictly lower A as the intra-chunk kernel solves it,
    over 16 x 16 blocks: the diagonal blocks by forward substitution (one column
    at a time), B_ik = -T_ii A_ik, then two dependent steps:
        T_10 = B_10 T_00, T_21 = B_21 T_11, T_32 = B_32 T_22,
        C_30 = B_30 + B_32 B_20, C_31 = B_31 + B_32 B_21;
        T_20 = B_20 T_00 + B_21 T_10, T_31 = B_31 T_11 + B_32 T_21,
        T_30 = C_30 T_00 + C_31 T_10."""
    n = 16
    blk = lambda M, i, j: M[n * i:n * (i + 1), n * j:n * (j + 1)]
    Tii = []
    for i in range(4):
        Ai = blk(A, i, i)
        Ti = np.zeros((n, n))
        for cl in range(n):
            t = np.zeros(n)
            t[cl] = 1.0
            for r in range(cl + 1, n):
                t[r] = -sum(Ai[r, k] * t[k] for k in range(r))
            Ti[:, cl] = t
        Tii.append(Ti)
    Bm = {(i, k): -Tii[i] @ blk(A, i, k) for i in range(4) for k in range(i)}
    T = {(i, i): Tii[i] for i in range(4)}
    T[1, 0] = Bm[1, 0] @ T[0, 0]
    T[2, 1] = Bm[2, 1] @ T[1, 1]
    T[3, 2] = Bm[3, 2] @ T[2, 2]
    C30 = Bm[3, 0] + Bm[3, 2] @ Bm[2, 0]
    C31 = Bm[3, 1] + Bm[3, 2] @ Bm[2, 1]
    T[2, 0] = Bm[2, 0] @ T[0, 0] + Bm[2, 1] @ T[1, 0]
    T[3, 1] = Bm[3, 1] @ T[1, 1] + Bm[3, 2] @ T[2, 1]
    T[3, 0] = C30 @ T[0, 0] + C31 @ T[1, 0]
    out = np.zeros((C, C))
    for (i, j), M in T.items():
        out[n * i:n * (i + 1), n * j:n * (j + 1)] = M
    return out


def test_blocked_two_step_inverse_matches_direct_inverse():
    # A = (P K^T) o Gamma- as the kernel forms it, from one chunk of the
    # generator's gates and keys
    (al, ml, be, et), inp = _chunk_gates(seed=9)
    k = np.asarray(inp.k, dtype=np.float64)[0, C:2 * C, 1]
    gam = _oracle_gamma(inp)
    gm = np.zeros((C, C))
    gm[1:, :] = gam[:-1, :]                      # Gamma-_{r,i} = Gamma_{r-1,i}
    A = np.tril(np.exp(al)[:, None] * (k @ k.T) * gm, -1)
    T = _blocked_inverse(A)
    ref = np.linalg.inv(np.eye(C) + A)
    assert np.abs(T - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    # the schedule leaves the strict upper triangle at zero and the diagonal at one
    assert np.all(np.triu(T, 1) == 0.0) and np.all(np.diag(T) == 1.0)


def test_blocked_two_step_inverse_catches_a_wrong_schedule():
    """The check above is sharp: dropping the B_32 B_20 term of C_30 (a
    plausible slip in the two-step schedule) moves T_30 far outside it."""
    rng = np.random.default_rng(3)
    A = np.tril(rng.standard_normal((C, C)) * 0.2, -1)
    ref = np.linalg.inv(np.eye(C) + A)
    T = _blocked_inverse(A)
    assert np.abs(T - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    n = 16
    B = lambda i, k: -np.linalg.inv(np.eye(n) + A[n * i:n * (i + 1), n * i:n * (i + 1)]) @ \
        A[n * i:n * (i + 1), n * k:n * (k + 1)]
    wrong30 = B(3, 0) @ T[:n, :n] + (B(3, 1) + B(3, 2) @ B(2, 1)) @ T[n:2 * n, :n]
    assert np.abs(wrong30 - ref[3 * n:, :n]).max() > 1e-3


def test_tensor_core_factorisation_matches_oracle():
    """The tensor-core path's factorisation, step by step, against the stepwise
    oracle over several chunks with non-zero entering states.  Per chunk the
    intra-chunk kernel forms Qhat = Q - d K, A = (P K^T) o Gamma-, T = (I + A)^-1,
    [T; Att T] with Att = (Qhat K^T) o Gamma, A2T = [K^T Diag(Gamma_C) T;
    -K^T Diag(w) T] (w_r = eta_r mubar_C / mubar_r) and the records alphabar_r,
    D2_r = alpha_r b_{r-1}, b_r; the chain then forms
        Y = V - (alphabar_r K S - D2_r K M),  [Vtilde; Att T Y] = [T; Att T] Y,
        o = alphabar_r Qhat S - b_r Qhat M + Att T Y,
        S <- alphabar_C S - b_C M + A2T_S Y,  M <- mubar_C M + A2T_M Y."""
    d, dcorr, NTc = 16, 0.5, 3
    inp = mi.make_inputs(mi.Spec("factor", B=1, T=NTc * C, H=1, d=d, dtype="f32",
                                 state_std=0.05, seed=11))
    q, k, v = (np.asarray(x, dtype=np.float64)[0, :, 0] for x in (inp.q, inp.k, inp.v))
    al, ml, be, et = (np.asarray(x, dtype=np.float64)[0, :, 0] for x in
                      (inp.alpha_log, inp.mu_log, inp.beta, inp.eta))
    _, _, _, gamma = oracle.chunk_coeffs(inp.alpha_log, inp.mu_log, inp.beta, inp.eta, C)
    S = np.asarray(inp.S0, dtype=np.float64)[0, 0].copy()
    M = np.asarray(inp.M0, dtype=np.float64)[0, 0].copy()
    o = np.zeros((NTc * C, d))
    vt = np.zeros((NTc * C, d))
    for n in range(NTc):
        sl = slice(n * C, (n + 1) * C)
        K, Q, V = k[sl], q[sl], v[sl]
        a, la, lm = np.exp(al[sl]), np.cumsum(al[sl]), np.cumsum(ml[sl])
        abar, mbar = np.exp(la), np.exp(lm)
        c = np.cumsum(be[sl] * mbar / abar)
        b = abar * c
        G = gamma[0, 0, n]
        Gm = np.zeros((C, C))
        Gm[1:, :] = G[:-1, :]
        A = np.tril(a[:, None] * (K @ K.T) * Gm, -1)
        T = np.linalg.inv(np.eye(C) + A)
        Qh = Q - dcorr * K
        Att = np.tril((Qh @ K.T) * G)
        w = et[sl] * mbar[-1] / mbar
        A2S = K.T @ (G[-1][:, None] * T)
        A2M = -K.T @ (w[:, None] * T)
        D2 = a * np.concatenate(([0.0], b[:-1]))
        Y = V - (abar[:, None] * (K @ S) - D2[:, None] * (K @ M))
        vt[sl] = T @ Y
        o[sl] = abar[:, None] * (Qh @ S) - b[:, None] * (Qh @ M) + (Att @ T) @ Y
        S, M = abar[-1] * S - b[-1] * M + A2S @ Y, mbar[-1] * M + A2M @ Y
    ro, rvt, rS, rM = oracle.chunk_fwd(inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log,
                                      inp.beta, inp.eta, dcorr, inp.S0, inp.M0)
    for x, ref in ((o, ro[0, :, 0]), (vt, rvt[0, :, 0]), (S, rS[0, 0]), (M, rM[0, 0])):
        assert np.abs(x - ref).max() <= 1e-9 * np.abs(ref).max()


def test_backward_blocked_column_recurrence():
    """The backward coefficient phase's R_{j,i} = sum_{r>=j} dG_{r,i} alphabar_r /
    alphabar_j, i.e. R_j = dG_j + alpha_{j+1} R_{j+1} down each column (rows
    j >= i), as the kernel runs it: four blocks of 16 rows, each from a zero
    carry keeping L_j and the decay P_j = alpha_{j+1} .. alpha_{16(p+1)} to its
    block's end, then the carries passed up from the blocks below and
    R_j = L_j + P_j carry."""
    rng = np.random.default_rng(5)
    al = rng.uniform(0.3, 1.0, C)
    dG = np.tril(rng.standard_normal((C, C)))
    al1 = np.append(al[1:], 0.0)                 # alpha_{j+1}; none past the chunk
    ref = np.zeros((C, C))
    for i in range(C):
        R = 0.0
        for j in range(C - 1, i - 1, -1):
            R = dG[j, i] + al1[j] * R
            ref[j, i] = R
    out = np.zeros((C, C))
    for i in range(C):
        Ls, Ps = [], []
        for part in range(4):
            lo = 16 * part
            L = np.array([dG[lo + e, i] if lo + e >= i else 0.0 for e in range(16)])
            P = np.zeros(16)
            l, pr = 0.0, 1.0
            for e in range(15, -1, -1):
                pr *= al1[lo + e]
                l = L[e] + al1[lo + e] * l
                L[e], P[e] = l, pr
            Ls.append(L)
            Ps.append(P)
        for part in range(4):
            carry = 0.0
            for q in range(3, part, -1):
                carry = Ls[q][0] + Ps[q][0] * carry
            for e in range(16):
                j = 16 * part + e
                if j >= i:
                    out[j, i] = Ls[part][e] + Ps[part][e] * carry
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()


def test_backward_affine_suffix_scan():
    """Rb_j = db_j + alpha_{j+1} Rb_{j+1} (Rb_C = 0) as a warp's suffix scan:
    lane l composes the maps of positions 2l, 2l+1 as (b0 + a0 b1, a0 a1), the
    lanes combine with the ones `off` above (off = 1, 2, 4, 8, 16) by
    (b, a) <- (b + a b', a a'), and position 2l+1 takes db + alpha Rb of 2l+2."""
    rng = np.random.default_rng(6)
    al = rng.uniform(0.3, 1.0, C)
    db = rng.standard_normal(C)
    ref = np.zeros(C)
    R = 0.0
    for j in range(C - 1, -1, -1):
        R = db[j] + (al[j + 1] if j + 1 < C else 0.0) * R
        ref[j] = R
    sb = np.zeros(32)
    sa = np.zeros(32)
    a1s = np.zeros(32)
    for lane in range(32):
        j0, j1 = 2 * lane, 2 * lane + 1
        a0, a1 = al[j1], (al[j1 + 1] if j1 + 1 < C else 0.0)
        sb[lane], sa[lane], a1s[lane] = a0 * db[j1] + db[j0], a0 * a1, a1
    off = 1
    while off < 32:
        ob = np.append(sb[off:], np.zeros(off))  # shuffle down: lane l reads lane l + off
        oa = np.append(sa[off:], np.zeros(off))
        live = np.arange(32) + off < 32
        sb = np.where(live, sb + sa * ob, sb)
        sa = np.where(live, sa * oa, sa)
        off <<= 1
    nxt = np.append(sb[1:], 0.0)
    out = np.zeros(C)
    out[0::2] = sb
    out[1::2] = db[1::2] + a1s * nxt
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max()


def test_backward_state_rebuild_from_saved_vtilde():
    """The backward pass keeps only Vtilde from the forward pass and rebuilds
    the chunk-entering states by the scan the state-rebuild kernel runs:
        D_S = K^T Diag(Gamma_{C,.}) Vtilde,  D_M = K^T Diag(w) Vtilde,
        S <- alphabar_C S - b_C M + D_S,     M <- mubar_C M - D_M.
    Each rebuilt state equals the oracle's state after that many tokens."""
    d, NTc = 16, 3
    inp = mi.make_inputs(mi.Spec("rebuild", B=1, T=NTc * C, H=1, d=d, dtype="f32",
                                 state_std=0.05, seed=12))
    args = (inp.alpha_log, inp.mu_log, inp.beta, inp.eta)
    _, vt, _, _ = oracle.chunk_fwd(inp.q, inp.k, inp.v, *args, inp.d_corr, inp.S0, inp.M0)
    _, _, _, gamma = oracle.chunk_coeffs(*args, C)
    k = np.asarray(inp.k, dtype=np.float64)[0, :, 0]
    al, ml, be, et = (np.asarray(x, dtype=np.float64)[0, :, 0] for x in args)
    S = np.asarray(inp.S0, dtype=np.float64)[0, 0].copy()
    M = np.asarray(inp.M0, dtype=np.float64)[0, 0].copy()
    for n in range(NTc):
        sl = slice(n * C, (n + 1) * C)
        la, lm = np.cumsum(al[sl]), np.cumsum(ml[sl])
        abar, mbar = np.exp(la), np.exp(lm)
        bC = abar[-1] * np.sum(be[sl] * mbar / abar)
        w = et[sl] * mbar[-1] / mbar
        V = vt[0, sl, 0]
        DS = k[sl].T @ (gamma[0, 0, n][-1][:, None] * V)
        DM = k[sl].T @ (w[:, None] * V)
        S, M = abar[-1] * S - bC * M + DS, mbar[-1] * M - DM
        T1 = (n + 1) * C
        cut = lambda x: None if x is None else np.asarray(x)[:, :T1]
        _, _, rS, rM = oracle.chunk_fwd(cut(inp.q), cut(inp.k), cut(inp.v),
                                        *(cut(g) for g in args), inp.d_corr, inp.S0, inp.M0)
        for x, ref in ((S, rS[0, 0]), (M, rM[0, 0])):
            assert np.abs(x - ref).max() <= 1e-10 * np.abs(ref).max()
