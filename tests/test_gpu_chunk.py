"""mdn_chunk_fwd on the GPU against the fp64 oracle, element by element
(rel-L2 over whole tensors, or over sampled heads at full workload size)."""
import zlib

import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from momentum_delta_rule_mdn_b200 import _lib
from parity import TOL, compare_all, compare_heads, config_inputs, oracle_all, rel_l2, to_np

pytestmark = pytest.mark.gpu


def run(inp, flags=0, **kw):
    dev = mi.to_torch(inp, "cuda")
    out = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"],
                        dev["beta"], dev["eta"], inp.d_corr, dev["S0"], dev["M0"], flags=flags,
                        **kw)
    torch.cuda.synchronize()
    return out


def all_heads(spec):
    return [(b, h) for b in range(spec.B) for h in range(spec.H)]


def test_config0_tiny_fp32():
    """B1 H1 T256 d64 fp32: the whole output against the oracle at rel-L2 <= 1e-4."""
    inp = config_inputs(0)
    errs = compare_heads(run(inp), inp, all_heads(inp.spec), TOL["f32"])
    print("config0 rel-L2 (o, vtilde, S_T, M_T):", errs)


SMALL = [
    # name, B, T, H, d, dtype, state_std  (T spans several chunks and a ragged tail)
    ("bf16_d128_ragged", 2, 200, 3, 128, "bf16", 0.01),
    ("bf16_d64_even", 1, 320, 2, 64, "bf16", 0.0),
    ("f32_d64_ragged", 1, 130, 2, 64, "f32", 0.05),
    ("f32_d128_ragged", 1, 100, 2, 128, "f32", 0.05),
    ("bf16_T1", 2, 1, 2, 128, "bf16", 0.01),
    ("bf16_T63", 1, 63, 2, 128, "bf16", 0.01),
    ("bf16_T65", 1, 65, 2, 128, "bf16", 0.01),
    ("f32_T64_exact", 1, 64, 1, 64, "f32", 0.0),
]


@pytest.mark.parametrize("name,B,T,H,d,dtype,std", SMALL, ids=[s[0] for s in SMALL])
def test_small_cases(name, B, T, H, d, dtype, std):
    inp = mi.make_inputs(mi.Spec(name, B=B, T=T, H=H, d=d, dtype=dtype, state_std=std,
                                 seed=zlib.crc32(name.encode()) % 1000 + 2000))
    compare_heads(run(inp), inp, all_heads(inp.spec), TOL[dtype])


@pytest.mark.parametrize("flags", [_lib.MDN_SLICE32, _lib.MDN_SLICE64, _lib.MDN_SLICE128])
@pytest.mark.parametrize("name,B,T,H", [("ragged", 2, 200, 3), ("T1", 1, 1, 2), ("T65", 1, 65, 1),
                                         ("long", 1, 1000, 2), ("many_heads", 3, 130, 60)])
def test_inter_slice_widths(name, B, T, H, flags):
    """Every chain width of the inter-chunk kernel against the oracle (180 heads:
    more chains than SMs, so the chains run in more than one wave)."""
    inp = mi.make_inputs(mi.Spec("slice_" + name, B=B, T=T, H=H, d=128, dtype="bf16",
                                 state_std=0.01, seed=zlib.crc32(name.encode()) % 1000 + 3000))
    compare_heads(run(inp, flags=flags), inp, all_heads(inp.spec), TOL["bf16"])


@pytest.mark.parametrize("flags", [0, _lib.MDN_FORCE_SIMT, _lib.MDN_SLICE32, _lib.MDN_SLICE64])
@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_full_size_configs_every_head(cfg, flags):
    """The workload configurations at full size, in the launch configuration the
    benchmark times (flags = 0), against the oracle over the whole batch: every
    head and every token of o, vtilde, S_T and M_T."""
    inp = config_inputs(cfg)
    out = run(inp, flags=flags)
    errs = compare_all(out, oracle_all(cfg), TOL["bf16"])
    for t in out:
        assert torch.isfinite(t.float()).all()
    print(f"config{cfg} flags={flags} rel-L2 (o, vtilde, S_T, M_T):",
          ", ".join(f"{e:.3e}" for e in errs))


@pytest.mark.parametrize("split", [128, 100])
def test_resume_equals_single_pass(split):
    """[0, split) then [split, T) with the first call's (S_T, M_T) as (S0, M0)."""
    spec = mi.Spec("resume", B=2, T=256, H=2, d=128, state_std=0.02, seed=31)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    g = {k: dev[k] for k in ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta")}
    full = mdn.chunk_fwd(*g.values(), inp.d_corr, dev["S0"], dev["M0"])
    a = mdn.chunk_fwd(*(t[:, :split].contiguous() for t in g.values()), inp.d_corr,
                      dev["S0"], dev["M0"])
    b = mdn.chunk_fwd(*(t[:, split:].contiguous() for t in g.values()), inp.d_corr, a[2], a[3])
    torch.cuda.synchronize()
    o = torch.cat([a[0], b[0]], 1)
    assert rel_l2(to_np(o), to_np(full[0])) <= 5e-3
    assert rel_l2(to_np(b[2]), to_np(full[2])) <= 5e-3
    assert rel_l2(to_np(b[3]), to_np(full[3])) <= 5e-3
    compare_heads((o, torch.cat([a[1], b[1]], 1), b[2], b[3]), inp, all_heads(spec), TOL["bf16"])


def test_states_may_alias_inputs():
    spec = mi.Spec("alias", B=1, T=128, H=2, d=64, dtype="f32", state_std=0.05, seed=32)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    S, M = dev["S0"].clone(), dev["M0"].clone()
    o = torch.empty_like(dev["q"])
    vt = torch.empty_like(o)
    mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"], dev["beta"],
                  dev["eta"], inp.d_corr, S, M, out=(o, vt, S, M))
    torch.cuda.synchronize()
    compare_heads((o, vt, S, M), inp, all_heads(spec), TOL["f32"])


def test_empty_sequence_copies_states():
    spec = mi.Spec("empty", B=2, T=0, H=2, d=128, state_std=0.1, seed=33)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    o, vt, S, M = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"],
                                dev["beta"], dev["eta"], 0.5, dev["S0"], dev["M0"])
    torch.cuda.synchronize()
    assert torch.equal(S, dev["S0"]) and torch.equal(M, dev["M0"])
    o, vt, S, M = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"],
                                dev["beta"], dev["eta"], 0.5)
    torch.cuda.synchronize()
    assert not S.any() and not M.any()


@pytest.mark.parametrize("kind", ["mu_tiny", "stress_alpha1_mu_clamp", "eta_small"])
def test_degenerate_gates(kind):
    """mu -> 0 (log mu = -30) approaches the gated delta rule; alpha -> 1 with mu at
    its clamp exercises Gamma where the log-broadcast form would cancel."""
    base = mi.Spec(kind, B=1, T=256, H=2, d=128, state_std=0.01, seed=41)
    if kind == "stress_alpha1_mu_clamp":
        base = mi.replace(base, a_mean=6.0, x_mean=-1.5, c_mean=-5.0)
    if kind == "eta_small":
        base = mi.replace(base, x_mean=-3.0)
    inp = mi.make_inputs(base)
    if kind == "mu_tiny":
        inp.mu_log[:] = -30.0
    compare_heads(run(inp), inp, all_heads(base), TOL["bf16"])


def test_check_finite_flag_reports_nan():
    spec = mi.Spec("nan", B=1, T=128, H=1, d=64, dtype="f32", seed=34)
    inp = mi.make_inputs(spec)
    assert run(inp, flags=_lib.MDN_CHECK_FINITE) is not None
    inp.v_store[0, 70, 0, 3] = np.nan
    with pytest.raises(mdn.MDNError) as e:
        run(inp, flags=_lib.MDN_CHECK_FINITE)
    assert e.value.status == _lib.MDN_ERR_NONFINITE


def test_host_tensors_round_trip():
    """The public call with host tensors: copies in, compute, copies out."""
    spec = mi.Spec("host", B=1, T=192, H=2, d=128, state_std=0.01, seed=35)
    inp = mi.make_inputs(spec)
    host = mi.to_torch(inp, "cpu", pin=True)
    out = mdn.chunk_fwd(host["q"], host["k"], host["v"], host["alpha_log"], host["mu_log"],
                        host["beta"], host["eta"], inp.d_corr, host["S0"], host["M0"])
    assert all(t.device.type == "cpu" for t in out)
    compare_heads(out, inp, all_heads(spec), TOL["bf16"])


def test_chunk_fwd_cuda_graph_replay():
    """The tensor-core pass captured in a CUDA graph (ready-flag reset, both
    kernels and their programmatic dependency) and replayed twice, the second
    time on new inputs written into the same buffers: each replay matches the
    oracle on its own inputs."""
    specs = [mi.Spec("graph_a", B=2, T=300, H=3, d=128, dtype="bf16", state_std=0.01, seed=4100),
             mi.Spec("graph_b", B=2, T=300, H=3, d=128, dtype="bf16", state_std=0.01, seed=4101)]
    inps = [mi.make_inputs(s) for s in specs]
    devs = [mi.to_torch(i, "cuda") for i in inps]
    names = ("q", "k", "v", "alpha_log", "mu_log", "beta", "eta", "S0", "M0")
    buf = {n: devs[0][n].clone() for n in names}
    B, T, H, d = 2, 300, 3, 128
    ws = torch.empty(mdn.chunk_fwd_workspace_size(B, T, H, d), dtype=torch.uint8, device="cuda")
    out = (torch.empty_like(buf["q"]), torch.empty_like(buf["q"]),
           torch.empty((B, H, d, d), device="cuda"), torch.empty((B, H, d, d), device="cuda"))

    def call():
        mdn.chunk_fwd(buf["q"], buf["k"], buf["v"], buf["alpha_log"], buf["mu_log"], buf["beta"],
                      buf["eta"], inps[0].d_corr, buf["S0"], buf["M0"], out=out, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()  # first use outside the capture (kernel attributes, tensor-map encoder)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    for r in range(2):
        for n in names:
            buf[n].copy_(devs[r][n])
        for t in out:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        compare_heads(out, inps[r], all_heads(inps[r].spec), TOL["bf16"])


@pytest.mark.parametrize("width", [0, _lib.MDN_SLICE128])
def test_timeout_path_reports_and_recovers(width):
    """Failure injected on the host: the intra-chunk kernel is not launched, so
    the inter-chunk kernel's bounded wait for the first chunk's operands runs
    out; its CTAs stop cleanly and the call reports MDN_ERR_TIMEOUT.  The
    context stays usable: the next normal call is correct.  Both chain kernels
    (32-column slices, chosen for these two heads, and one CTA per head)."""
    inp = mi.make_inputs(mi.Spec("timeout", B=1, T=130, H=2, d=128, dtype="bf16",
                                 state_std=0.01, seed=4200))
    with pytest.raises(mdn.MDNError) as err:
        run(inp, flags=_lib.MDN_TEST_NO_INTRA | _lib.MDN_CHECK_FINITE | width)
    assert err.value.status == _lib.MDN_ERR_TIMEOUT
    compare_heads(run(inp), inp, all_heads(inp.spec), TOL["bf16"])
    # without MDN_CHECK_FINITE the call returns at once; the status query reports
    # the expired wait afterwards, and a normal call on the same workspace clears it
    dev = mi.to_torch(inp, "cuda")
    B, T, H, d = inp.spec.B, inp.spec.T, inp.spec.H, inp.spec.d
    ws = torch.empty(mdn.chunk_fwd_workspace_size(B, T, H, d), dtype=torch.uint8, device="cuda")
    args = (dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"], dev["beta"],
            dev["eta"], inp.d_corr, dev["S0"], dev["M0"])
    mdn.chunk_fwd(*args, workspace=ws, flags=_lib.MDN_TEST_NO_INTRA | width)
    assert mdn.chunk_fwd_status(ws) == _lib.MDN_ERR_TIMEOUT
    out = mdn.chunk_fwd(*args, workspace=ws, flags=width)
    assert mdn.chunk_fwd_status(ws) == _lib.MDN_OK
    compare_heads(out, inp, all_heads(inp.spec), TOL["bf16"])
