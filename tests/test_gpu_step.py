"""mdn_step (decode) on the GPU against the oracle recurrence."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from parity import TOL, config_inputs, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _seq_to_steps(t):
    """[B,T,H,...] -> [T,B,H,...] contiguous, so step t is a contiguous slice."""
    return t.transpose(0, 1).contiguous()


@pytest.mark.parametrize("dtype,d,B,H", [
    ("f32", 64, 2, 3), ("f32", 128, 2, 3), ("bf16", 64, 2, 3), ("bf16", 128, 2, 3),
    # head counts at which the kernel splits d_v into 32 and 64 columns per block
    ("bf16", 128, 10, 8), ("bf16", 128, 40, 8), ("f32", 64, 10, 16), ("f32", 64, 40, 8),
])
def test_step_small(dtype, d, B, H):
    spec = mi.Spec("step_small", B=B, T=24 if B * H < 50 else 4, H=H, d=d, dtype=dtype,
                   state_std=0.05, seed=77)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    S, M = dev["S0"].clone(), dev["M0"].clone()
    steps = {k: _seq_to_steps(dev[k]) for k in ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")}
    o_ref, vt_ref, S_ref, M_ref = oracle.chunk_fwd(inp.q, inp.k, inp.v, inp.alpha_log,
                                                   inp.mu_log, inp.beta, inp.eta, inp.d_corr,
                                                   inp.S0, inp.M0)
    os_, vts = [], []
    for t in range(spec.T):
        o, vt = mdn.step(*(steps[k][t] for k in ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")),
                         inp.d_corr, S, M)
        os_.append(to_np(o))
        vts.append(to_np(vt))
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == "f32" else TOL["bf16"]
    assert rel_l2(np.stack(os_, 1), o_ref) <= tol
    assert rel_l2(np.stack(vts, 1), vt_ref) <= tol
    assert rel_l2(to_np(S), S_ref) <= tol
    assert rel_l2(to_np(M), M_ref) <= tol


@pytest.fixture(scope="module")
def decode_cfg():
    return config_inputs(4)


def test_step_decode_config_every_head(decode_cfg):
    """512 consecutive mdn_step calls at B=256, H=16, d=128 (bf16); every head
    against the oracle recurrence (one oracle call over the whole batch)."""
    inp = decode_cfg
    dev = mi.to_torch(inp, "cuda")
    B, T, H, d = inp.q.shape
    S = torch.zeros((B, H, d, d), device="cuda")
    M = torch.zeros_like(S)
    steps = {k: _seq_to_steps(dev[k]) for k in ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")}
    o_all = torch.empty((T, B, H, d), dtype=torch.bfloat16, device="cuda")
    vt_all = torch.empty_like(o_all)
    for t in range(T):
        mdn.step(*(steps[k][t] for k in ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")),
                 inp.d_corr, S, M, o=o_all[t], vtilde=vt_all[t])
    torch.cuda.synchronize()
    o_np, vt_np, S_np, M_np = to_np(o_all), to_np(vt_all), to_np(S), to_np(M)
    ro, rvt, rS, rM = oracle.chunk_fwd(inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta,
                                       inp.eta, inp.d_corr)
    errs = [rel_l2(o_np, ro.transpose(1, 0, 2, 3)), rel_l2(vt_np, rvt.transpose(1, 0, 2, 3)),
            rel_l2(S_np, rS), rel_l2(M_np, rM)]
    print("decode 512 steps rel-L2 (o, vtilde, S, M):", ", ".join(f"{e:.3e}" for e in errs))
    assert max(errs) <= TOL["bf16"], errs
    # the same 512-token sequence through the chunkwise pass ("training == inference")
    o_c, vt_c, S_c, M_c = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"],
                                        dev["mu_log"], dev["beta"], dev["eta"], inp.d_corr)
    torch.cuda.synchronize()
    assert rel_l2(to_np(o_c).transpose(1, 0, 2, 3), o_np) <= TOL["bf16"]
    assert rel_l2(to_np(vt_c).transpose(1, 0, 2, 3), vt_np) <= TOL["bf16"]
    assert rel_l2(to_np(S_c), S_np) <= TOL["bf16"]
    assert rel_l2(to_np(M_c), M_np) <= TOL["bf16"]


def test_step_without_vtilde_and_empty():
    spec = mi.Spec("step_nv", B=1, T=1, H=2, d=128, state_std=0.1, seed=5)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    S, M = dev["S0"].clone(), dev["M0"].clone()
    g = lambda k: dev[k][:, 0].contiguous()
    o, vt = mdn.step(g("q"), g("k"), g("v"), g("alpha_log"), g("mu_log"), g("beta"), g("eta"),
                     inp.d_corr, S, M, want_vtilde=False)
    assert vt is None
    ro, _, rS, _ = oracle.step(inp.q[:, 0], inp.k[:, 0], inp.v[:, 0], inp.alpha_log[:, 0],
                               inp.mu_log[:, 0], inp.beta[:, 0], inp.eta[:, 0], inp.d_corr,
                               inp.S0, inp.M0)
    assert rel_l2(to_np(o), ro) <= TOL["bf16"]
    assert rel_l2(to_np(S), rS) <= 1e-5
    e = lambda *s: torch.empty(s, device="cuda")
    mdn.step(e(0, 2, 64).bfloat16(), e(0, 2, 64).bfloat16(), e(0, 2, 64).bfloat16(), e(0, 2),
             e(0, 2), e(0, 2), e(0, 2), 0.5, e(0, 2, 64, 64), e(0, 2, 64, 64))
