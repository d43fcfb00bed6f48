"""mdn_chunk_bwd (the backward pass from the saved Vtilde) on the GPU against
the fp64 gradient oracle."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
from oracle import backward as ob
import momentum_delta_rule_mdn_b200 as mdn
from parity import rel_l2, to_np

pytestmark = pytest.mark.gpu

GATES = ("alpha_log", "mu_log", "beta", "eta")
NAMES = ("dq", "dk", "dv", "dalpha_log", "dmu_log", "dbeta", "deta", "dS0", "dM0")
# rel-L2 bars: fp32 storage (the saved Vtilde exact to fp32) and bf16 storage
# (q, k, v, Vtilde and the cotangent of o rounded to bf16; fp32 arithmetic)
TOL = {"f32": 1e-5, "bf16": 1e-2}


def _run(spec, cot_seed=7, with_state_cot=True):
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    o, vt, S_T, M_T = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES),
                                    inp.d_corr, dev["S0"], dev["M0"])
    rng = np.random.default_rng(cot_seed)
    B, T, H, d = inp.q.shape
    do = rng.standard_normal((B, T, H, d)).astype(np.float32)
    if spec.dtype == "bf16":
        do = mi.bf16_bits_to_f32(mi.bf16_round_bits(do))
    dS = rng.standard_normal((B, H, d, d)).astype(np.float32) if with_state_cot else None
    dM = rng.standard_normal((B, H, d, d)).astype(np.float32) if with_state_cot else None
    tdev = lambda x: None if x is None else torch.from_numpy(x).cuda()
    do_dev = tdev(do).to(dev["q"].dtype)
    g = mdn.chunk_bwd(dev["q"], dev["k"], dev["v"], *(dev[x] for x in GATES), inp.d_corr, vt,
                      do_dev, dev["S0"], dev["M0"], tdev(dS), tdev(dM))
    torch.cuda.synchronize()
    ref = ob.chunk_bwd(inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta, inp.eta,
                       inp.d_corr, inp.S0, inp.M0, do, dS, dM)
    return g, ref


@pytest.mark.parametrize("dtype,d,T", [("f32", 64, 200), ("f32", 128, 130),
                                       ("bf16", 128, 200), ("bf16", 64, 64)])
def test_bwd_matches_gradient_oracle(dtype, d, T):
    """Several chunks and a ragged last one, non-zero entering states and all
    three cotangents."""
    spec = mi.Spec("bwd", B=1, T=T, H=2, d=d, dtype=dtype, state_std=0.05, seed=501)
    g, ref = _run(spec)
    errs = {}
    for n in NAMES:
        got = to_np(g[n])
        assert np.all(np.isfinite(got)), n
        errs[n] = rel_l2(got, ref[n])
    print(f"bwd {dtype} d={d} T={T} rel-L2:", " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= TOL[dtype], (n, e)


def test_bwd_layer_shape_sampled():
    """The layer workload's head shape (d = 128, bf16) over 512 tokens, B = 2,
    H = 2, zero entering states, o's cotangent only."""
    spec = mi.Spec("bwd_layer", B=2, T=512, H=2, d=128, seed=502)
    g, ref = _run(spec, with_state_cot=False)
    errs = {n: rel_l2(to_np(g[n]), ref[n]) for n in NAMES}
    print("bwd layer shape B2 T512 H2 rel-L2:", " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= TOL["bf16"], (n, e)


def test_bwd_zero_length_passes_state_cotangents():
    B, H, d = 2, 3, 64
    e = lambda *s: torch.empty(s, device="cuda")
    z = lambda *s: torch.zeros(s, device="cuda")
    dS, dM = torch.randn(B, H, d, d, device="cuda"), torch.randn(B, H, d, d, device="cuda")
    g = mdn.chunk_bwd(e(B, 0, H, d), e(B, 0, H, d), e(B, 0, H, d), *(z(B, 0, H) for _ in range(4)),
                      0.5, e(B, 0, H, d), e(B, 0, H, d), None, None, dS, dM)
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], dS) and torch.equal(g["dM0"], dM)


def test_bwd_layer_workload_sampled_heads():
    """The whole layer workload (B = 4, T = 2048, H = 8, d = 128, bf16) through the
    forward and backward passes; two heads against the oracle."""
    inp = mi.make_inputs(mi.WORKLOADS[1])
    dev = mi.to_torch(inp, "cuda")
    o, vt, _, _ = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES),
                                inp.d_corr)
    rng = np.random.default_rng(11)
    do = mi.bf16_bits_to_f32(mi.bf16_round_bits(rng.standard_normal(inp.q.shape).astype(np.float32)))
    g = mdn.chunk_bwd(dev["q"], dev["k"], dev["v"], *(dev[x] for x in GATES), inp.d_corr, vt,
                      torch.from_numpy(do).cuda().to(torch.bfloat16))
    torch.cuda.synchronize()
    got = {n: to_np(g[n]) for n in NAMES}
    for (b, h) in [(0, 0), (3, 5)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref = ob.chunk_bwd(inp.q[sl], inp.k[sl], inp.v[sl], inp.alpha_log[sl], inp.mu_log[sl],
                           inp.beta[sl], inp.eta[sl], inp.d_corr, None, None, do[sl])
        errs = {}
        for n in NAMES:
            mine = got[n][b:b + 1, :, h:h + 1] if n not in ("dS0", "dM0") else got[n][b:b + 1, h:h + 1]
            errs[n] = rel_l2(mine, ref[n])
        print(f"bwd layer400m head ({b},{h}) rel-L2:", " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
        for n, e in errs.items():
            assert e <= TOL["bf16"], (b, h, n, e)


def test_bwd_long_sequence_long_memory():
    """64 chunks with the long-context gates (alpha and mu close to 1, as in the
    16K-context workload): the state rebuild carries each chunk's increment
    (stored in bf16) far down the sequence, so its rounding would build up
    here if anywhere.  B = H = 1, T = 4096, d = 128, bf16, against the fp64
    gradient oracle."""
    spec = mi.Spec("bwd_long", B=1, T=4096, H=1, d=128, a_mean=3.0, c_mean=3.0,
                   state_std=0.01, seed=506)
    g, ref = _run(spec)
    errs = {n: rel_l2(to_np(g[n]), ref[n]) for n in NAMES}
    print("bwd long memory T4096 rel-L2:", " ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= TOL["bf16"], (n, e)


def test_bwd_cuda_graph_replay_matches_eager():
    """The backward call (which forks the state rebuild onto a side stream and
    joins it back) captured in a CUDA graph and replayed gives the eager
    results bit for bit."""
    spec = mi.Spec("bwd_graph", B=1, T=320, H=3, d=128, state_std=0.02, seed=503)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    o, vt, _, _ = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES),
                                inp.d_corr, dev["S0"], dev["M0"])
    do = torch.randn_like(o)
    args = (dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES), inp.d_corr, vt, do,
            dev["S0"], dev["M0"])
    eager = mdn.chunk_bwd(*args)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        mdn.chunk_bwd(*args)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        got = mdn.chunk_bwd(*args)
    graph.replay()
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(got[n], eager[n]), n


def test_bwd_tensor_core_path_matches_cuda_core_path():
    """bf16, d = 128: the tcgen05 kernels (reverse chain, its operands, the
    state scan, both product kernels) against the fp32 CUDA-core kernels on the
    same inputs and the same saved Vtilde."""
    from momentum_delta_rule_mdn_b200 import _lib
    spec = mi.Spec("bwd_paths", B=2, T=300, H=3, d=128, state_std=0.03, seed=504)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    o, vt, _, _ = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES),
                                inp.d_corr, dev["S0"], dev["M0"])
    do = torch.randn_like(o)
    dS = torch.randn(2, 3, 128, 128, device="cuda")
    args = (dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES), inp.d_corr, vt, do,
            dev["S0"], dev["M0"], dS, None)
    tc = mdn.chunk_bwd(*args, flags=_lib.MDN_CHECK_FINITE)
    simt = mdn.chunk_bwd(*args, flags=_lib.MDN_CHECK_FINITE | _lib.MDN_FORCE_SIMT)
    for n in NAMES:
        e = rel_l2(to_np(tc[n]), to_np(simt[n]))
        assert e <= 1e-2, (n, e)
