"""K-0 (gates from pre-activations) and the decode step's ||Delta S||_F on the
GPU, against the oracle."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from parity import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _gates_close(got, ref):
    """Elementwise bar.  The log-domain outputs to 4e-6 of (1 + |ref|); beta and
    eta to 4e-6 relative, widened by the oracle's own rounding where it forms
    tanh(x) + 1 in fp64: that sum cancels for very negative x, leaving an
    absolute error of about 1.1e-16 in eta (twice that, relatively, in beta,
    which goes as eta^2 there)."""
    al, ml, be, et = (to_np(t).astype(np.float64) for t in got)
    ral, rml, rbe, ret = ref
    for x in (al, ml, be, et):
        assert np.all(np.isfinite(x))
    assert np.max(np.abs(al - ral) / (1.0 + np.abs(ral)), initial=0) < 4e-6
    assert np.max(np.abs(ml - rml) / (1.0 + np.abs(rml)), initial=0) < 4e-6
    cancel = 2.3e-16 / np.maximum(ret, 1e-300)
    assert np.all(np.abs(et - ret) <= (4e-6 + cancel) * ret + 1e-37)
    assert np.all(np.abs(be - rbe) <= (4e-6 + 2 * cancel) * rbe + 1e-37)


def _dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda() for a in arrs]


@pytest.mark.parametrize("act", ["tanh", "2sigmoid"])
@pytest.mark.parametrize("cfg", [1, 3])
def test_gate_params_workload_preactivations(act, cfg):
    """The pre-activations of the workloads ([B,T,H], n % 4 == 0: the float4 path)."""
    spec = mi.replace(mi.WORKLOADS[cfg], B=2, T=1000, H=mi.WORKLOADS[cfg].H)
    inp = mi.make_inputs(spec)
    pre = (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)
    got = mdn.gate_params(*_dev(*pre), s=spec.eta_scale, mu_log_min=spec.mu_log_min,
                          eta_act=act)
    torch.cuda.synchronize()
    ref = oracle.gates(*pre, s=spec.eta_scale, mu_log_min=spec.mu_log_min, eta_act=act)
    _gates_close(got, ref)


@pytest.mark.parametrize("n", [0, 1, 3, 1001, 4096 * 37 + 2])
@pytest.mark.parametrize("s,mu_min", [(1.0, -2.0), (0.25, -1.0), (4.0, -1.357)])
def test_gate_params_ragged_sizes_and_scales(n, s, mu_min):
    """n not a multiple of 4 (the scalar path), several grid-stride rounds."""
    rng = np.random.default_rng(n + 7)
    pre = [rng.standard_normal(n) * 3.0 for _ in range(4)]
    got = mdn.gate_params(*_dev(*pre), s=s, mu_log_min=mu_min)
    torch.cuda.synchronize()
    pre32 = [p.astype(np.float32) for p in pre]
    _gates_close(got, oracle.gates(*pre32, s=s, mu_log_min=mu_min))


def test_gate_params_misaligned_views_take_the_scalar_path():
    rng = np.random.default_rng(3)
    base = [torch.from_numpy(rng.standard_normal(4097).astype(np.float32)).cuda()
            for _ in range(4)]
    pre = [t[1:] for t in base]                 # 4-byte but not 16-byte aligned
    outs = [torch.empty(4097, device="cuda")[1:] for _ in range(4)]
    got = mdn.gate_params(*pre, s=1.5, mu_log_min=-2.0, out=tuple(outs))
    torch.cuda.synchronize()
    _gates_close(got, oracle.gates(*(to_np(t) for t in pre), s=1.5, mu_log_min=-2.0))


@pytest.mark.parametrize("act", ["tanh", "2sigmoid"])
def test_gate_params_extreme_preactivations(act):
    """Saturated pre-activations stay finite (alpha_log may be -inf only where
    cos^2(theta) sigmoid(a) underflows in fp64 too) and match the oracle."""
    vals = np.array([-100.0, -40.0, -17.0, -5.0, -1e-3, 0.0, 1e-3, 5.0, 17.0, 40.0, 100.0])
    g = np.stack(np.meshgrid(vals, vals, vals, vals, indexing="ij"), 0).reshape(4, -1)
    got = mdn.gate_params(*_dev(*g), s=2.0, mu_log_min=-2.0, eta_act=act)
    torch.cuda.synchronize()
    ref = oracle.gates(*g.astype(np.float32), s=2.0, mu_log_min=-2.0, eta_act=act)
    al, ml, be, et = (to_np(t).astype(np.float64) for t in got)
    assert np.all(np.isfinite(al)) and np.all(np.isfinite(be))
    assert np.all((be >= 0) & (be <= 1)) and np.all((et >= 0) & (et <= 2))
    assert np.all(ml >= -2.0) and np.all(ml <= 0)
    assert np.max(np.abs(et - ref[3])) < 1e-6
    assert np.max(np.abs(al - ref[0]) / (1.0 + np.abs(ref[0]))) < 4e-6
    assert np.max(np.abs(ml - ref[1])) < 4e-6
    assert np.max(np.abs(be - ref[2])) < 1e-6
    # away from fp32 underflow the relative bar holds as well
    sel = (ref[2] > 1e-30) & (ref[3] > 1e-30)
    _gates_close([torch.from_numpy(x[sel].astype(np.float32)) for x in (al, ml, be, et)],
                 [r[sel] for r in ref])


def test_gate_params_feed_the_chunk_pass():
    """K-0's gates drive mdn_chunk_fwd to the oracle's result from the same
    pre-activations (the oracle forms its gates itself)."""
    spec = mi.replace(mi.WORKLOADS[1], B=1, T=320, H=4)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    pre = (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)
    al, ml, be, et = mdn.gate_params(*_dev(*pre), s=spec.eta_scale, mu_log_min=spec.mu_log_min)
    o, vt, S_T, M_T = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], al, ml, be, et, inp.d_corr)
    torch.cuda.synchronize()
    ral, rml, rbe, ret = oracle.gates(*pre, s=spec.eta_scale, mu_log_min=spec.mu_log_min)
    ro, rvt, rS, rM = oracle.chunk_fwd(inp.q, inp.k, inp.v, ral, rml, rbe, ret, inp.d_corr)
    for g, r in ((o, ro), (vt, rvt), (S_T, rS), (M_T, rM)):
        assert rel_l2(to_np(g), r) <= TOL["bf16"]


def _steps(t):
    return t.transpose(0, 1).contiguous()


@pytest.mark.parametrize("dtype,d,B,H", [("f32", 64, 2, 3), ("bf16", 128, 2, 3),
                                         ("bf16", 128, 40, 8), ("f32", 128, 10, 8)])
def test_step_delta_norm_matches_oracle(dtype, d, B, H):
    """||S_t - S_{t-1}||_F per head and step, against the oracle's fp64 states;
    o, vtilde and the states match mdn_step's."""
    T = 6
    spec = mi.Spec("step_dnorm", B=B, T=T, H=H, d=d, dtype=dtype, state_std=0.05, seed=91)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    S, M = dev["S0"].clone(), dev["M0"].clone()
    S2, M2 = dev["S0"].clone(), dev["M0"].clone()
    keys = ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")
    st = {k: _steps(dev[k]) for k in keys}
    rS, rM = inp.S0.astype(np.float64), inp.M0.astype(np.float64)
    tol = 1e-5 if dtype == "f32" else TOL["bf16"]
    for t in range(T):
        args = [st[k][t] for k in keys]
        o, vt, dn = mdn.step_with_delta_norm(*args, inp.d_corr, S, M)
        o2, vt2 = mdn.step(*args, inp.d_corr, S2, M2)
        torch.cuda.synchronize()
        tok = [np.ascontiguousarray(getattr(inp, k)[:, t]) for k in keys]
        _, _, rS_new, rM_new = oracle.step(*tok, inp.d_corr, rS, rM)
        ref = oracle.step_delta_norm(rS, rS_new)
        got = to_np(dn)
        assert got.shape == (B, H)
        assert np.max(np.abs(got - ref) / ref) < (1e-4 if dtype == "f32" else 5e-3)
        # the norm is an extra output only: everything else is bit-identical
        assert torch.equal(o, o2) and torch.equal(vt, vt2)
        assert torch.equal(S, S2) and torch.equal(M, M2)
        rS, rM = rS_new, rM_new
    assert rel_l2(to_np(S), rS) <= tol


def test_step_delta_norm_of_a_still_state_is_zero():
    """alpha = 1, beta = 0: S does not move, so the norm is exactly 0."""
    B, H, d = 3, 4, 64
    z = lambda *s: torch.zeros(s, device="cuda")
    q = torch.randn(B, H, d, device="cuda")
    k = torch.nn.functional.normalize(torch.randn(B, H, d, device="cuda"), dim=-1)
    v = torch.randn(B, H, d, device="cuda")
    S = torch.randn(B, H, d, d, device="cuda")
    M = torch.randn(B, H, d, d, device="cuda")
    S0 = S.clone()
    _, _, dn = mdn.step_with_delta_norm(q, k, v, z(B, H), z(B, H) - 0.5, z(B, H),
                                        torch.ones(B, H, device="cuda"), 0.5, S, M)
    torch.cuda.synchronize()
    assert torch.equal(S, S0)
    assert torch.count_nonzero(dn).item() == 0


def test_step_delta_norm_decode_workload():
    """The decode workload's shape (B = 256, H = 16, d = 128, bf16): one token from
    random states; every head's norm against the oracle's fp64 step."""
    spec = mi.replace(mi.WORKLOADS[4], T=1, state_std=0.02, seed=1204)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    keys = ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")
    tok = {k: dev[k][:, 0].contiguous() for k in keys}
    S, M = dev["S0"].clone(), dev["M0"].clone()
    _, _, dn = mdn.step_with_delta_norm(*(tok[k] for k in keys), inp.d_corr, S, M)
    torch.cuda.synchronize()
    _, _, S1, _ = oracle.step(*(np.ascontiguousarray(getattr(inp, k)[:, 0]) for k in keys),
                              inp.d_corr, inp.S0, inp.M0)
    ref = oracle.step_delta_norm(inp.S0, S1)
    got = to_np(dn)
    assert np.max(np.abs(got - ref) / ref) < 5e-3
