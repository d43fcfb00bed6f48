"""fp64 gradients of the MDN forward pass (plain PyTorch autograd on the CPU).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline arm may use it.

What it differentiates ("MDN: Parallelizing Stepwise Momentum for Delta
Linear Attention"; paper.rainbus.top summary, steps 1 and 7; ijyty.com
article, sections 3 and 6): per head, token by token,

    p_t      = alpha_t k_t,             alpha_t = exp(alpha_log_t)
    vtilde_t = v_t - S_{t-1}^T p_t
    M_t      = mu_t M_{t-1} - eta_t k_t vtilde_t^T,   mu_t = exp(mu_log_t)
    S_t      = alpha_t S_{t-1} - beta_t M_t
    o_t      = S_t^T (q_t - d k_t)

The loss is L = <do, o> + <dS_T, S_T> + <dM_T, M_T> for given cotangents, so
its gradients are the vector-Jacobian products a backward pass returns.  The
pages' training method saves vtilde and rebuilds S, M from it (summary,
step 7; article, section 6); that is a way to compute these same numbers,
which are unique, so the oracle is the plain definition differentiated by
autograd.  ``forward`` is the same recurrence in torch, checked against the C
oracle by the pins; the pins also check the gradients against central
finite differences and a hand-derived single-token case.
"""
from __future__ import annotations

import numpy as np
import torch

_DT = torch.float64


def _t(x, requires_grad=False):
    t = torch.as_tensor(np.asarray(x, dtype=np.float64), dtype=_DT).clone()
    return t.requires_grad_(requires_grad)


def forward(q, k, v, alpha_log, mu_log, beta, eta, d: float, S0=None, M0=None):
    """The recurrence over [B,T,H,d] torch tensors (fp64).  Returns
    (o, vtilde, S_T, M_T) as torch tensors, differentiable."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = S0 if S0 is not None else torch.zeros((B, H, dk, dv), dtype=_DT)
    M = M0 if M0 is not None else torch.zeros((B, H, dk, dv), dtype=_DT)
    os_, vts = [], []
    for t in range(T):
        qt, kt, vt_in = q[:, t], k[:, t], v[:, t]                # [B,H,d]
        a = torch.exp(alpha_log[:, t])[..., None, None]          # [B,H,1,1]
        mu = torch.exp(mu_log[:, t])[..., None, None]
        be = beta[:, t][..., None, None]
        et = eta[:, t][..., None, None]
        p = a[..., 0] * kt                                       # [B,H,dk]
        vtil = vt_in - torch.einsum("bhij,bhi->bhj", S, p)
        M = mu * M - et * kt[..., :, None] * vtil[..., None, :]
        S = a * S - be * M
        qh = qt - d * kt
        os_.append(torch.einsum("bhij,bhi->bhj", S, qh))
        vts.append(vtil)
    o = torch.stack(os_, 1) if T else torch.zeros((B, 0, H, dv), dtype=_DT)
    vt = torch.stack(vts, 1) if T else torch.zeros((B, 0, H, dv), dtype=_DT)
    return o, vt, S, M


def chunk_bwd(q, k, v, alpha_log, mu_log, beta, eta, d: float, S0=None, M0=None,
              do=None, dS_T=None, dM_T=None):
    """Gradients of <do, o> + <dS_T, S_T> + <dM_T, M_T> (any cotangent may be
    None = zero).  Inputs as for the forward pass ([B,T,H,d], gates [B,T,H],
    states [B,H,d,d]).  Returns a dict of fp64 numpy arrays: dq, dk, dv,
    dalpha_log, dmu_log, dbeta, deta, dS0, dM0."""
    names = ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")
    x = {n: _t(a, True) for n, a in zip(names, (q, k, v, alpha_log, mu_log, beta, eta))}
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    S0t = _t(S0 if S0 is not None else np.zeros((B, H, dk, dv)), True)
    M0t = _t(M0 if M0 is not None else np.zeros((B, H, dk, dv)), True)
    o, _, S_T, M_T = forward(*(x[n] for n in names), d, S0t, M0t)
    loss = torch.zeros((), dtype=_DT)
    if do is not None:
        loss = loss + (o * _t(do)).sum()
    if dS_T is not None:
        loss = loss + (S_T * _t(dS_T)).sum()
    if dM_T is not None:
        loss = loss + (M_T * _t(dM_T)).sum()
    leaves = [x[n] for n in names] + [S0t, M0t]
    if not loss.requires_grad:
        grads = [torch.zeros_like(t) for t in leaves]
    else:
        grads = torch.autograd.grad(loss, leaves, allow_unused=True)
        grads = [torch.zeros_like(t) if g is None else g for g, t in zip(grads, leaves)]
    keys = ("dq", "dk", "dv", "dalpha_log", "dmu_log", "dbeta", "deta", "dS0", "dM0")
    return {k_: g.detach().numpy() for k_, g in zip(keys, grads)}


def loss_value(q, k, v, alpha_log, mu_log, beta, eta, d: float, S0=None, M0=None,
               do=None, dS_T=None, dM_T=None) -> float:
    """The scalar whose gradients chunk_bwd returns (for finite differences)."""
    with torch.no_grad():
        S0t = None if S0 is None else _t(S0)
        M0t = None if M0 is None else _t(M0)
        o, _, S_T, M_T = forward(*(_t(a) for a in (q, k, v, alpha_log, mu_log, beta, eta)),
                                 d, S0t, M0t)
        val = 0.0
        if do is not None:
            val += float((o * _t(do)).sum())
        if dS_T is not None:
            val += float((S_T * _t(dS_T)).sum())
        if dM_T is not None:
            val += float((M_T * _t(dM_T)).sum())
        return val
