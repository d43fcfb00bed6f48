"""Helpers shared by the GPU parity tests: seeded inputs on the device, the
oracle on selected heads, and the rel-L2 metric the tolerances are stated in."""
from __future__ import annotations

import functools

import numpy as np
import torch

import mdn_inputs as mi
import oracle

# rel-L2 bounds: fp32 inputs 1e-4; bf16 inputs with fp32 state 2e-2.
TOL = {"f32": 1e-4, "bf16": 2e-2}


@functools.lru_cache(maxsize=None)
def config_inputs(i: int) -> mi.Inputs:
    """The i-th workload's inputs, generated once per test session."""
    return mi.make_inputs(mi.WORKLOADS[i])


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_inputs(inp: mi.Inputs, device="cuda"):
    return mi.to_torch(inp, device)


def oracle_heads(inp: mi.Inputs, heads, T0: int = 0, T1=None, S0=None, M0=None):
    """Oracle forward pass on the listed (b, h) heads over tokens [T0, T1).
    Returns lists of per-head (o [T,d], vt [T,d], S_T [d,d], M_T [d,d])."""
    T1 = inp.spec.T if T1 is None else T1
    outs = []
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(T0, T1), slice(h, h + 1))
        s0 = None if S0 is None else S0[b:b + 1, h:h + 1]
        m0 = None if M0 is None else M0[b:b + 1, h:h + 1]
        o, vt, S, M = oracle.chunk_fwd(inp.q[sl], inp.k[sl], inp.v[sl], inp.alpha_log[sl],
                                       inp.mu_log[sl], inp.beta[sl], inp.eta[sl],
                                       inp.d_corr, s0, m0)
        outs.append((o[0, :, 0], vt[0, :, 0], S[0, 0], M[0, 0]))
    return outs


def compare_heads(got, inp: mi.Inputs, heads, tol: float, T0: int = 0, T1=None,
                  S0=None, M0=None):
    """got = (o, vt, S_T, M_T) device tensors over the whole batch; compares the
    listed heads with the oracle; returns the four rel-L2 errors."""
    if S0 is None and inp.S0 is not None:
        S0, M0 = inp.S0, inp.M0
    ref = oracle_heads(inp, heads, T0, T1, S0, M0)
    o, vt, S, M = (to_np(t) for t in got)
    errs = []
    for idx, name in enumerate(("o", "vtilde", "S_T", "M_T")):
        g, r = [], []
        for (b, h), rh in zip(heads, ref):
            if idx < 2:
                g.append((o if idx == 0 else vt)[b, :, h])
            else:
                g.append((S if idx == 2 else M)[b, h])
            r.append(rh[idx])
        errs.append(rel_l2(np.stack(g), np.stack(r)))
    names = ("o", "vtilde", "S_T", "M_T")
    bad = [f"{n}: rel-L2 {e:.3e}" for n, e in zip(names, errs) if not e <= tol]
    assert not bad, f"{bad} > {tol:.1e}; all: {dict(zip(names, errs))}"
    return errs


@functools.lru_cache(maxsize=3)
def oracle_all(i: int):
    """The oracle over the whole batch of the i-th workload (parallel over heads),
    computed once per test session."""
    inp = config_inputs(i)
    return oracle.chunk_fwd(inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta, inp.eta,
                            inp.d_corr, inp.S0, inp.M0)


def compare_all(got, ref, tol: float):
    """got = (o, vt, S_T, M_T) device tensors, ref = the oracle's four arrays for
    the same batch: every head, every token.  Returns the four rel-L2 errors."""
    names = ("o", "vtilde", "S_T", "M_T")
    errs = [rel_l2(to_np(g), r) for g, r in zip(got, ref)]
    bad = [f"{n}: rel-L2 {e:.3e}" for n, e in zip(names, errs) if not e <= tol]
    assert not bad, f"{bad} > {tol:.1e}; all: {dict(zip(names, errs))}"
    return errs
