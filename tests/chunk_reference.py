"""Test-only fp64 restatement of the chunkwise MDN forward pass.

Plain numpy, no log domain, small sizes only.  It restates "MDN: Parallelizing
Stepwise Momentum for Delta Linear Attention" (paper.rainbus.top summary,
steps 2-4): within each chunk of C tokens (all cumulative products restart at
the chunk start; S, M are the states entering the chunk)

  alphabar_r = prod_{j<=r} alpha_j,  mubar_r = prod_{j<=r} mu_j
  c_r = sum_{j<=r} beta_j mubar_j / alphabar_j,     b_r = alphabar_r c_r
  Gamma_{r,i} = eta_i (alphabar_r / mubar_i) (c_r - c_{i-1})   (i <= r)
  Gamma-_{r,i} = Gamma_{r-1,i}                                 (i <  r)
  P = Diag(alpha) K,  T = (I + (P K^T) o Gamma-)^{-1}
  U = T V,  Y = T Diag(alphabar_{r-1}) P,  Z = T Diag(b_{r-1}) P
  Vtilde = U - Y S + Z M
  O = Diag(alphabar) Qhat S - Diag(b) Qhat M + ((Qhat K^T) o Gamma) Vtilde
  S' = alphabar_L S - b_L M + K^T Diag(Gamma_{L,:}) Vtilde
  M' = mubar_L M - K^T Diag(eta_i mubar_L / mubar_i) Vtilde

The eta_i factor on write i, the "previous step" reading of the index range
0..C-1 in Y and Z, and the chunk-end state update and output formula are
readings of the pages (they are not printed there); the CPU
tests pin this restatement to the stepwise oracle for several C.
It is independent of the oracle and of the CUDA library.
"""
from __future__ import annotations

import numpy as np


def chunk_forward(q, k, v, alpha_log, mu_log, beta, eta, d, S0=None, M0=None, C=64):
    """[B,T,H,d] inputs -> fp64 (o, vtilde, S_T, M_T)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    al, ml, be, et = (np.asarray(x, dtype=np.float64) for x in (alpha_log, mu_log, beta, eta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    vt = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    M_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            M = np.zeros((dk, dv)) if M0 is None else np.array(M0[b, h], dtype=np.float64)
            for n0 in range(0, T, C):
                sl = slice(n0, min(T, n0 + C))
                K, V, Q = k[b, sl, h], v[b, sl, h], q[b, sl, h]
                L = K.shape[0]
                alpha = np.exp(al[b, sl, h])
                abar = np.exp(np.cumsum(al[b, sl, h]))
                mbar = np.exp(np.cumsum(ml[b, sl, h]))
                c = np.cumsum(be[b, sl, h] * mbar / abar)
                c_prev = np.concatenate([[0.0], c[:-1]])
                bcoef = abar * c
                abar_prev = np.concatenate([[1.0], abar[:-1]])
                b_prev = np.concatenate([[0.0], bcoef[:-1]])
                e = et[b, sl, h]
                G = np.tril(e[None, :] * abar[:, None] / mbar[None, :]
                            * (c[:, None] - c_prev[None, :]))
                Gm = np.zeros_like(G)
                Gm[1:, :] = G[:-1, :]
                P = alpha[:, None] * K
                A = (P @ K.T) * Gm
                Tm = np.linalg.inv(np.eye(L) + A)
                U = Tm @ V
                Y = Tm @ (abar_prev[:, None] * P)
                Z = Tm @ (b_prev[:, None] * P)
                Vt = U - Y @ S + Z @ M
                Qh = Q - d * K
                O = (abar[:, None] * (Qh @ S) - bcoef[:, None] * (Qh @ M)
                     + ((Qh @ K.T) * G) @ Vt)
                S_new = abar[-1] * S - bcoef[-1] * M + K.T @ (G[-1][:, None] * Vt)
                M_new = mbar[-1] * M - K.T @ ((e * mbar[-1] / mbar)[:, None] * Vt)
                o[b, sl, h] = O
                vt[b, sl, h] = Vt
                S, M = S_new, M_new
            S_T[b, h], M_T[b, h] = S, M
    return o, vt, S_T, M_T


def chunk_backward(q, k, v, alpha_log, mu_log, beta, eta, d, S0=None, M0=None,
                   do=None, dS_T=None, dM_T=None, C=64):
    """Gradients of <do, o> + <dS_T, S_T> + <dM_T, M_T> through the chunk form
    above, chunk by chunk in reverse: the state adjoints (dS, dM) are carried
    backwards like S, M are carried forwards; every other gradient is local to
    its chunk, given the chunk's entering states and the adjoints leaving it.
    Gate gradients go through the adjoints of the chunk coefficients
    (alphabar, b, Gamma, the chunk-end scalars) and their definitions.
    Returns a dict like the gradient oracle's."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    al, ml, be, et = (np.asarray(x, dtype=np.float64) for x in (alpha_log, mu_log, beta, eta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    z = lambda *s: np.zeros(s)
    g = dict(dq=z(B, T, H, dk), dk=z(B, T, H, dk), dv=z(B, T, H, dv),
             dalpha_log=z(B, T, H), dmu_log=z(B, T, H), dbeta=z(B, T, H), deta=z(B, T, H),
             dS0=z(B, H, dk, dv), dM0=z(B, H, dk, dv))
    do = z(B, T, H, dv) if do is None else np.asarray(do, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            # forward: the states entering every chunk
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            M = np.zeros((dk, dv)) if M0 is None else np.array(M0[b, h], dtype=np.float64)
            starts = list(range(0, T, C))
            entering = []
            for n0 in starts:
                entering.append((S, M))
                cf = _coeffs(q, k, v, al, ml, be, et, d, b, h, n0, min(T, n0 + C), S, M)
                S, M = cf["S_new"], cf["M_new"]
            dS = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T[b, h], dtype=np.float64)
            dM = np.zeros((dk, dv)) if dM_T is None else np.array(dM_T[b, h], dtype=np.float64)
            for n0, (S, M) in reversed(list(zip(starts, entering))):
                n1 = min(T, n0 + C)
                cf = _coeffs(q, k, v, al, ml, be, et, d, b, h, n0, n1, S, M)
                dS, dM = _chunk_bwd(cf, do[b, n0:n1, h], dS, dM, d, g, b, h, n0, n1)
            g["dS0"][b, h], g["dM0"][b, h] = dS, dM
    return g


def _coeffs(q, k, v, al, ml, be, et, d, b, h, n0, n1, S, M):
    sl = slice(n0, n1)
    K, V, Q = k[b, sl, h], v[b, sl, h], q[b, sl, h]
    L = K.shape[0]
    la, lm = np.cumsum(al[b, sl, h]), np.cumsum(ml[b, sl, h])
    alpha, abar, mbar = np.exp(al[b, sl, h]), np.exp(la), np.exp(lm)
    beta, e = be[b, sl, h], et[b, sl, h]
    # Gamma without eta, by its expanded definition (ratios of cumulative products)
    Gp = np.zeros((L, L))
    for r in range(L):
        for i in range(r + 1):
            Gp[r, i] = sum(np.exp(la[r] - la[j]) * beta[j] * np.exp(lm[j] - lm[i])
                           for j in range(i, r + 1))
    G = Gp * e[None, :]
    bcoef = np.array([sum(np.exp(la[r] - la[j]) * beta[j] * mbar[j] for j in range(r + 1))
                      for r in range(L)])
    b_prev = np.concatenate([[0.0], bcoef[:-1]])
    Gm = np.zeros_like(G)
    Gm[1:, :] = G[:-1, :]
    P = alpha[:, None] * K
    Tm = np.linalg.inv(np.eye(L) + (P @ K.T) * Gm)
    D1, D2 = abar, b_prev * alpha            # alphabar_{r-1} alpha_r = alphabar_r
    Yv = V - D1[:, None] * (K @ S) + D2[:, None] * (K @ M)
    Vt = Tm @ Yv
    Qh = Q - d * K
    w = e * mbar[-1] / mbar
    return dict(K=K, Q=Q, Qh=Qh, L=L, la=la, lm=lm, alpha=alpha, abar=abar, mbar=mbar,
                beta=beta, e=e, G=G, Gp=Gp, Gm=Gm, bcoef=bcoef, b_prev=b_prev, P=P, Tm=Tm,
                D1=D1, D2=D2, Yv=Yv, Vt=Vt, w=w, S=S, M=M,
                S_new=abar[-1] * S - bcoef[-1] * M + K.T @ (G[-1][:, None] * Vt),
                M_new=mbar[-1] * M - K.T @ (w[:, None] * Vt))


def _chunk_bwd(cf, dO, dS, dM, d, g, b, h, n0, n1):
    K, Qh, Vt, Tm, G, Gm, P = cf["K"], cf["Qh"], cf["Vt"], cf["Tm"], cf["G"], cf["Gm"], cf["P"]
    S, M, L = cf["S"], cf["M"], cf["L"]
    abar, bcoef, mbar, D1, D2, w = cf["abar"], cf["bcoef"], cf["mbar"], cf["D1"], cf["D2"], cf["w"]
    la, lm, alpha, beta, e = cf["la"], cf["lm"], cf["alpha"], cf["beta"], cf["e"]
    gL = G[-1]
    QK = Qh @ K.T
    KdS, KdM = K @ dS, K @ dM
    # state adjoints through the chunk
    dVt = (QK * G).T @ dO + gL[:, None] * KdS - w[:, None] * KdM
    dYv = Tm.T @ dVt
    dS_prev = abar[-1] * dS + Qh.T @ (abar[:, None] * dO) - K.T @ (D1[:, None] * dYv)
    dM_prev = (-bcoef[-1] * dS + mbar[-1] * dM - Qh.T @ (bcoef[:, None] * dO)
               + K.T @ (D2[:, None] * dYv))
    # token gradients
    dOV = dO @ Vt.T
    dQh = abar[:, None] * (dO @ S.T) - bcoef[:, None] * (dO @ M.T) + (dOV * G) @ K
    dA = -(dYv @ Vt.T) * np.tri(L, L, -1)                            # A is strictly lower
    dPK = dA * Gm
    dP = dPK @ K
    dK = ((dOV * G).T @ Qh + gL[:, None] * (Vt @ dS.T) - w[:, None] * (Vt @ dM.T)
          - D1[:, None] * (dYv @ S.T) + D2[:, None] * (dYv @ M.T) + dPK.T @ P
          + alpha[:, None] * dP)
    g["dq"][b, n0:n1, h] = dQh
    g["dk"][b, n0:n1, h] = dK - d * dQh
    g["dv"][b, n0:n1, h] = dYv
    # adjoints of the chunk coefficients
    d_abar = np.sum(dO * (Qh @ S), 1) - np.sum(dYv * (K @ S), 1)     # O and D1
    d_b = -np.sum(dO * (Qh @ M), 1)
    dD2 = np.sum(dYv * (K @ M), 1)
    d_alpha = np.sum(dP * K, 1) + dD2 * cf["b_prev"]                  # P and D2 (d/d alpha)
    d_b[:-1] += (dD2 * alpha)[1:]                                      # D2_r = b_{r-1} alpha_r
    dG = dOV * QK * (np.tril(np.ones((L, L))))
    dG[:-1, :] += (dA * (P @ K.T))[1:, :]                              # Gamma-_{r,i} = Gamma_{r-1,i}
    dG[-1, :] += np.sum(Vt * KdS, 1)                                   # Gamma_{L,i} in S'
    dw = -np.sum(Vt * KdM, 1)
    d_abar[-1] += np.sum(S * dS)
    d_b[-1] += -np.sum(M * dS)
    d_mbar_last = np.sum(M * dM)
    # to log-domain cumulative sums la, lm and the direct gates
    dla = d_abar * abar + d_b * bcoef
    dlm = np.zeros(L)
    dlm[-1] += d_mbar_last * mbar[-1] + np.sum(dw * w)
    dlm -= dw * w
    de = dw * mbar[-1] / mbar                                          # w_r = eta_r mbar_L / mbar_r
    dbeta = np.zeros(L)
    for r in range(L):
        for j in range(r + 1):
            t = np.exp(la[r] - la[j]) * beta[j] * mbar[j] * d_b[r]    # b_r = sum_j ...
            dbeta[j] += np.exp(la[r] - la[j]) * mbar[j] * d_b[r]
            dla[j] -= t
            dlm[j] += t
    GdG = dG * G
    dla += GdG.sum(1)
    dlm -= GdG.sum(0)
    de += (dG * cf["Gp"]).sum(0)
    for j in range(L):
        U = 0.0
        for r in range(j, L):
            for i in range(j + 1):
                U += dG[r, i] * e[i] * np.exp(la[r] - la[j]) * np.exp(lm[j] - lm[i])
        dbeta[j] += U
        dla[j] -= beta[j] * U
        dlm[j] += beta[j] * U
    rev = lambda x: np.cumsum(x[::-1])[::-1]
    g["dalpha_log"][b, n0:n1, h] = d_alpha * alpha + rev(dla)
    g["dmu_log"][b, n0:n1, h] = rev(dlm)
    g["dbeta"][b, n0:n1, h] = dbeta
    g["deta"][b, n0:n1, h] = de
    return dS_prev, dM_prev
