"""Seeded synthetic inputs for the MDN forward pass and the decode step.

This module is shared by the tests, the benchmark and every caller of the
oracle.  It holds no part of the recurrence or of its chunkwise form: it only
draws q, k, v, the four gates and the entering states with the shapes and
value distributions of the workloads, and rounds the stored values to their
storage dtype (bf16 by round-to-nearest-even, done once, here).

Gate synthesis follows the stable gating parameterisation of "MDN:
Parallelizing Stepwise Momentum for Delta Linear Attention" (paper.rainbus.top
summary, step 6; ijyty.com article, section 5): eta = tanh(x) + 1,
theta = arctan(eta * s), alpha = cos^2(theta) * sigmoid(a),
beta = sin^2(theta) * sigmoid(b), log mu = max(logsigmoid(c), mu_log_min).
The kernels take the resulting gates as given and never clamp them.

Draw order for one input set (one numpy Generator seeded with ``spec.seed``):
q, k, v (float32 normals, [B,T,H,d]), x_eta, a, b, c (float64 normals,
[B,T,H]), then S0, M0 (float32, [B,H,d,d]) when ``state_std > 0``.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import numpy as np

__all__ = ["Spec", "Inputs", "WORKLOADS", "make_inputs", "bf16_round_bits",
           "bf16_bits_to_f32", "replace"]


@dataclass(frozen=True)
class Spec:
    """Shape, storage dtype and gate distribution of one synthetic workload."""
    name: str
    B: int
    T: int
    H: int
    d: int                      # d_k = d_v
    dtype: str = "bf16"         # storage dtype of q, k, v (and of o, v_tilde)
    C: int = 64                 # chunk length used by the chunkwise kernels
    a_mean: float = 0.0         # mean of the alpha pre-activation a
    b_mean: float = 0.0         # mean of the beta pre-activation b
    c_mean: float = 0.0         # mean of the mu pre-activation c
    x_mean: float = 0.0         # mean of the eta pre-activation x
    eta_scale: float = 1.0      # s in theta = arctan(eta * s)
    mu_log_min: float = -1.0    # lower clamp of log mu
    state_std: float = 0.0      # > 0: S0, M0 ~ N(0, state_std^2); 0: zero states
    q_corr: float = 0.5         # the output-correction scalar d in q_hat = q - d k
    seed: int = 1000
    decode: bool = False        # the T tokens are fed one mdn_step call at a time


# The five workloads.  Index i uses seed 1000 + i.
WORKLOADS = [
    Spec("tiny_fp32_B1_H1_T256_d64", B=1, T=256, H=1, d=64, dtype="f32", seed=1000),
    Spec("layer400m_B4_H8_T2048_d128", B=4, T=2048, H=8, d=128, seed=1001),
    Spec("layer1p3b_B8_H16_T4096_d128", B=8, T=4096, H=16, d=128, state_std=0.01,
         seed=1002),
    Spec("longctx_B1_H16_T16384_d128", B=1, T=16384, H=16, d=128, a_mean=3.0,
         c_mean=3.0, seed=1003),
    Spec("decode_B256_H16_d128_x512", B=256, T=512, H=16, d=128, decode=True,
         seed=1004),
]


def replace(spec: Spec, **kw) -> Spec:
    return dataclasses.replace(spec, **kw)


@dataclass
class Inputs:
    """One input set.

    ``q, k, v`` are float32 arrays holding exactly the stored values (for
    bf16 storage: the rounded values, upcast).  ``q_store`` etc. are what a
    device buffer holds: uint16 bf16 bit patterns, or float32.
    """
    spec: Spec
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_store: np.ndarray
    k_store: np.ndarray
    v_store: np.ndarray
    alpha_log: np.ndarray
    mu_log: np.ndarray
    beta: np.ndarray
    eta: np.ndarray
    S0: Optional[np.ndarray]
    M0: Optional[np.ndarray]
    # the gate pre-activations as float32 (what a gate-parameterisation kernel
    # reads); the gates above were formed from their float64 draws
    x_eta: Optional[np.ndarray] = None
    a_pre: Optional[np.ndarray] = None
    b_pre: Optional[np.ndarray] = None
    c_pre: Optional[np.ndarray] = None

    @property
    def d_corr(self) -> float:
        return self.spec.q_corr


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _logsigmoid(x: np.ndarray) -> np.ndarray:
    return -np.logaddexp(0.0, -x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return np.exp(_logsigmoid(x))


def make_inputs(spec: Spec) -> Inputs:
    rng = np.random.default_rng(spec.seed)
    B, T, H, d = spec.B, spec.T, spec.H, spec.d
    shape = (B, T, H, d)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    x = rng.standard_normal((B, T, H)) + spec.x_mean
    a = rng.standard_normal((B, T, H)) + spec.a_mean
    b = rng.standard_normal((B, T, H)) + spec.b_mean
    c = rng.standard_normal((B, T, H)) + spec.c_mean
    S0 = M0 = None
    if spec.state_std > 0:
        S0 = (rng.standard_normal((B, H, d, d)) * spec.state_std).astype(np.float32)
        M0 = (rng.standard_normal((B, H, d, d)) * spec.state_std).astype(np.float32)

    # k is L2-normalised per token before it is stored.
    if T > 0:
        norm = np.sqrt(np.einsum("bthi,bthi->bth", k, k, dtype=np.float64))
        k = (k / norm[..., None].astype(np.float32)).astype(np.float32)

    if spec.dtype == "bf16":
        q_store, k_store, v_store = (bf16_round_bits(t) for t in (q, k, v))
        q, k, v = (bf16_bits_to_f32(t) for t in (q_store, k_store, v_store))
    elif spec.dtype == "f32":
        q_store, k_store, v_store = q, k, v
    else:
        raise ValueError(f"unknown storage dtype {spec.dtype!r}")

    eta = np.tanh(x) + 1.0
    theta = np.arctan(eta * spec.eta_scale)
    alpha = np.cos(theta) ** 2 * _sigmoid(a)
    beta = np.sin(theta) ** 2 * _sigmoid(b)
    mu_log = np.maximum(_logsigmoid(c), spec.mu_log_min)
    f32 = np.float32
    return Inputs(spec=spec, q=q, k=k, v=v, q_store=q_store, k_store=k_store,
                  v_store=v_store, alpha_log=np.log(alpha).astype(f32),
                  mu_log=mu_log.astype(f32), beta=beta.astype(f32),
                  eta=eta.astype(f32), S0=S0, M0=M0, x_eta=x.astype(f32),
                  a_pre=a.astype(f32), b_pre=b.astype(f32), c_pre=c.astype(f32))


def to_torch(inp: Inputs, device="cpu", pin: bool = False) -> dict:
    """The stored input buffers as torch tensors (bf16 storage -> torch.bfloat16)."""
    import torch

    def conv(a: np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        if pin:
            t = t.pin_memory()
        return t.to(device) if device != "cpu" else t

    out = dict(q=conv(inp.q_store), k=conv(inp.k_store), v=conv(inp.v_store),
               alpha_log=conv(inp.alpha_log), mu_log=conv(inp.mu_log),
               beta=conv(inp.beta), eta=conv(inp.eta),
               S0=None if inp.S0 is None else conv(inp.S0),
               M0=None if inp.M0 is None else conv(inp.M0))
    return out
