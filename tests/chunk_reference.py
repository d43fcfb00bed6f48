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
this build's readings of the pages (they are not printed there); the CPU
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
