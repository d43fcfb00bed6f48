"""mdn_chunk_fwd_preact: the chunk pass with the gate parameterisation fused
into it (the gates computed from their pre-activations inside the kernels that
read them), against the oracle's gate parameterisation followed by the oracle's
recurrence, and against the two-call path (gate kernel, then the pass)."""
import zlib

import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from momentum_delta_rule_mdn_b200 import _lib
from parity import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, T, H, d, dtype, flags, eta_act, s, mu_log_min
    ("bf16_tc_tanh", 2, 300, 3, 128, "bf16", 0, "tanh", 1.0, -2.0),
    ("bf16_tc_2sig", 1, 257, 4, 128, "bf16", 0, "2sigmoid", 1.3, -1.357),
    ("bf16_simt", 1, 200, 2, 128, "bf16", _lib.MDN_FORCE_SIMT, "tanh", 0.7, -1.0),
    ("f32_d64", 1, 256, 1, 64, "f32", 0, "tanh", 1.0, -2.0),
    ("f32_d128_2sig", 1, 130, 2, 128, "f32", 0, "2sigmoid", 2.0, -1.5),
]


@pytest.mark.parametrize("name,B,T,H,d,dtype,flags,act,s,mu_min", CASES, ids=[c[0] for c in CASES])
def test_fused_gates_match_oracle(name, B, T, H, d, dtype, flags, act, s, mu_min):
    spec = mi.Spec(name, B=B, T=T, H=H, d=d, dtype=dtype, state_std=0.01,
                   seed=zlib.crc32(name.encode()) % 1000 + 6000)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    pre = [torch.from_numpy(np.ascontiguousarray(p, dtype=np.float32)).cuda()
           for p in (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)]
    got = mdn.chunk_fwd_preact(dev["q"], dev["k"], dev["v"], *pre, s=s, mu_log_min=mu_min,
                               eta_act=act, d=inp.d_corr, S0=dev["S0"], M0=dev["M0"],
                               flags=flags)
    torch.cuda.synchronize()
    # the oracle: its own gate parameterisation (fp64) of the same fp32
    # pre-activations, then its stepwise recurrence
    pre32 = [np.asarray(p, dtype=np.float32) for p in (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)]
    al, ml, be, et = oracle.gates(*pre32, s=s, mu_log_min=mu_min, eta_act=act)
    ref = oracle.chunk_fwd(inp.q, inp.k, inp.v, al, ml, be, et, inp.d_corr, inp.S0, inp.M0)
    tol = TOL[dtype]
    errs = [rel_l2(to_np(g), r) for g, r in zip(got, ref)]
    assert max(errs) <= tol, f"rel-L2 (o, vtilde, S_T, M_T) {errs} > {tol}"
    # the two-call path: the same gates through the gate kernel, then the pass
    gates = mdn.gate_params(*pre, s=s, mu_log_min=mu_min, eta_act=act)
    two = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *gates, inp.d_corr, dev["S0"], dev["M0"],
                        flags=flags)
    torch.cuda.synchronize()
    for g, t in zip(got, two):
        assert rel_l2(to_np(g), to_np(t)) <= (1e-5 if dtype == "f32" else 2e-3)
    print(name, "rel-L2 vs oracle:", ", ".join(f"{e:.2e}" for e in errs))


def test_fused_gates_full_size_layer1p3b():
    """The 1.3B-layer workload through the fused pass: its pre-activations with
    the workload's own s and clamp reproduce the workload's gates, so the result
    is checked against the oracle of the workload itself (every head)."""
    from parity import config_inputs, oracle_all, compare_all
    inp = config_inputs(2)
    spec = inp.spec
    dev = mi.to_torch(inp, "cuda")
    pre = [torch.from_numpy(np.ascontiguousarray(p, dtype=np.float32)).cuda()
           for p in (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)]
    got = mdn.chunk_fwd_preact(dev["q"], dev["k"], dev["v"], *pre, s=spec.eta_scale,
                               mu_log_min=spec.mu_log_min, eta_act="tanh", d=inp.d_corr,
                               S0=dev["S0"], M0=dev["M0"])
    torch.cuda.synchronize()
    errs = compare_all(got, oracle_all(2), TOL["bf16"])
    print("layer1p3b fused gates rel-L2:", ", ".join(f"{e:.2e}" for e in errs))
