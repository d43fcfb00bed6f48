"""fp64 CPU oracle for the MDN forward pass and decode step (ctypes binding).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package.  The CUDA
library and its Python binding never import it, and it imports nothing from
them.

The C source (``mdn_oracle.c``) runs the stepwise momentum recurrence of "MDN:
Parallelizing Stepwise Momentum for Delta Linear Attention" (paper.rainbus.top
summary, step 1; ijyty.com article, sections 3 and 6) in fp64, one token at a
time.  This module compiles it with gcc on first use and marshals numpy
arrays.  Inputs are upcast to fp64 exactly (the stored bf16/fp32 values).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "mdn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(_BUILD_DIR, "libmdn_oracle.so")
_lock = threading.Lock()
_libs: dict = {}


def compile_oracle(source: str = SOURCE, out: str = LIB_PATH) -> str:
    """Compile ``source`` into the shared library ``out`` (gcc, -O2, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-Wall", "-Wextra", "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def build() -> str:
    """Build the default oracle library if it is missing or older than its source."""
    with _lock:
        if (not os.path.exists(LIB_PATH)
                or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE)):
            compile_oracle()
    return LIB_PATH


_D = ctypes.POINTER(ctypes.c_double)


def _bind(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    i = ctypes.c_int
    lib.mdn_oracle_chunk_fwd.argtypes = [_D, _D, _D, _D, _D, _D, _D, ctypes.c_double,
                                         _D, _D, i, i, i, i, i, _D, _D, _D, _D]
    lib.mdn_oracle_chunk_fwd.restype = i
    lib.mdn_oracle_step.argtypes = [_D, _D, _D, _D, _D, _D, _D, ctypes.c_double,
                                    _D, _D, i, i, i, i, _D, _D]
    lib.mdn_oracle_step.restype = i
    lib.mdn_oracle_chunk_coeffs.argtypes = [_D, _D, _D, _D, i, i, i, i, _D, _D, _D, _D]
    lib.mdn_oracle_chunk_coeffs.restype = i
    lib.mdn_oracle_gates.argtypes = [_D, _D, _D, _D, ctypes.c_ssize_t, ctypes.c_double,
                                     ctypes.c_double, i, _D, _D, _D, _D]
    lib.mdn_oracle_gates.restype = i
    lib.mdn_oracle_max_threads.argtypes = []
    lib.mdn_oracle_max_threads.restype = i
    return lib


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """The oracle library at ``path`` (default: the built-in one, built on demand)."""
    path = path or build()
    with _lock:
        if path not in _libs:
            _libs[path] = _bind(path)
        return _libs[path]


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_D)


def max_threads(lib: Optional[ctypes.CDLL] = None) -> int:
    return int((lib or load()).mdn_oracle_max_threads())


def chunk_fwd(q, k, v, alpha_log, mu_log, beta, eta, d, S0=None, M0=None,
              lib: Optional[ctypes.CDLL] = None):
    """Forward pass over [B,T,H,d] inputs.  Returns fp64 (o, vtilde, S_T, M_T)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    al, ml, be, et = (_f64(x) for x in (alpha_log, mu_log, beta, eta))
    for g in (al, ml, be, et):
        assert g.shape == (B, T, H), g.shape
    S0 = None if S0 is None else _f64(S0)
    M0 = None if M0 is None else _f64(M0)
    o = np.empty((B, T, H, dv))
    vt = np.empty((B, T, H, dv))
    S_T = np.empty((B, H, dk, dv))
    M_T = np.empty((B, H, dk, dv))
    rc = lib.mdn_oracle_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(al), _ptr(ml),
                                  _ptr(be), _ptr(et), float(d), _ptr(S0), _ptr(M0),
                                  B, T, H, dk, dv, _ptr(o), _ptr(vt), _ptr(S_T), _ptr(M_T))
    if rc != 0:
        raise RuntimeError(f"mdn_oracle_chunk_fwd failed ({rc})")
    return o, vt, S_T, M_T


def chunk_fwd_varlen(q, k, v, alpha_log, mu_log, beta, eta, cu_seqlens, d, S0=None, M0=None,
                     lib: Optional[ctypes.CDLL] = None):
    """N sequences packed along the token axis: q, k, v [total_T,H,d], gates
    [total_T,H], cu_seqlens [N+1] (sequence s = tokens cu[s]:cu[s+1]), S0, M0
    [N,H,d,d] or None.  The pages run one sequence per batch row; packing is
    the plain extension, each sequence its own recurrence from its own
    entering state.  Returns fp64 (o, vtilde, S_T, M_T)."""
    cu = [int(x) for x in np.asarray(cu_seqlens)]
    N = len(cu) - 1
    total_T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    assert N >= 0 and cu[0] == 0 and cu[-1] == total_T
    assert all(cu[i] <= cu[i + 1] for i in range(N))
    o = np.zeros((total_T, H, dv))
    vt = np.zeros((total_T, H, dv))
    S_T = np.empty((N, H, dk, dv))
    M_T = np.empty((N, H, dk, dv))
    for s in range(N):
        a, b = cu[s], cu[s + 1]
        seq = lambda x: np.asarray(x)[a:b][None]
        st = lambda x: None if x is None else np.asarray(x)[s:s + 1]
        ro, rvt, rS, rM = chunk_fwd(seq(q), seq(k), seq(v), seq(alpha_log), seq(mu_log),
                                    seq(beta), seq(eta), d, st(S0), st(M0), lib=lib)
        o[a:b], vt[a:b], S_T[s], M_T[s] = ro[0], rvt[0], rS[0], rM[0]
    return o, vt, S_T, M_T


def step(q, k, v, alpha_log, mu_log, beta, eta, d, S, M,
         lib: Optional[ctypes.CDLL] = None):
    """One decode token over [B,H,d] inputs.  Returns fp64 (o, vtilde, S_new, M_new);
    the given S and M are not modified."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, dk = q.shape
    dv = v.shape[-1]
    al, ml, be, et = (_f64(x) for x in (alpha_log, mu_log, beta, eta))
    S = np.array(S, dtype=np.float64, order="C", copy=True)
    M = np.array(M, dtype=np.float64, order="C", copy=True)
    o = np.empty((B, H, dv))
    vt = np.empty((B, H, dv))
    rc = lib.mdn_oracle_step(_ptr(q), _ptr(k), _ptr(v), _ptr(al), _ptr(ml), _ptr(be),
                             _ptr(et), float(d), _ptr(S), _ptr(M), B, H, dk, dv,
                             _ptr(o), _ptr(vt))
    if rc != 0:
        raise RuntimeError(f"mdn_oracle_step failed ({rc})")
    return o, vt, S, M


def chunk_coeffs(alpha_log, mu_log, beta, eta, C: int, with_gamma: bool = True,
                 lib: Optional[ctypes.CDLL] = None):
    """Per-chunk (la, lm, lc [B,H,T], gamma [B,H,NT,C,C] or None), chunk-local."""
    lib = lib or load()
    al, ml, be, et = (_f64(x) for x in (alpha_log, mu_log, beta, eta))
    B, T, H = al.shape
    NT = (T + C - 1) // C
    la = np.empty((B, H, T))
    lm = np.empty((B, H, T))
    lc = np.empty((B, H, T))
    gamma = np.empty((B, H, NT, C, C)) if with_gamma else None
    rc = lib.mdn_oracle_chunk_coeffs(_ptr(al), _ptr(ml), _ptr(be), _ptr(et), B, T, H, C,
                                     _ptr(la), _ptr(lm), _ptr(lc), _ptr(gamma))
    if rc != 0:
        raise RuntimeError(f"mdn_oracle_chunk_coeffs failed ({rc})")
    return la, lm, lc, gamma


def gates(x_eta, a, b, c, s: float = 1.0, mu_log_min: float = -1.0, eta_act: str = "tanh",
          lib: Optional[ctypes.CDLL] = None):
    """Gates from pre-activations (any equal shapes).  Returns fp64
    (alpha_log, mu_log, beta, eta)."""
    lib = lib or load()
    x, aa, bb, cc = (_f64(t) for t in (x_eta, a, b, c))
    assert x.shape == aa.shape == bb.shape == cc.shape
    out = [np.empty(x.shape) for _ in range(4)]
    act = {"tanh": 0, "2sigmoid": 1}[eta_act]
    rc = lib.mdn_oracle_gates(_ptr(x), _ptr(aa), _ptr(bb), _ptr(cc), x.size, float(s),
                              float(mu_log_min), act, *(_ptr(o) for o in out))
    if rc != 0:
        raise RuntimeError(f"mdn_oracle_gates failed ({rc})")
    return tuple(out)


def step_delta_norm(S_old, S_new) -> np.ndarray:
    """Frobenius norm of the fast-weight change of one decode step, per head:
    ||S_t - S_{t-1}||_F (ijyty.com article, section 8)."""
    dS = np.asarray(S_new, dtype=np.float64) - np.asarray(S_old, dtype=np.float64)
    return np.sqrt((dS * dS).sum(axis=(-2, -1)))
