"""mdn_chunk_fwd_varlen (sequences packed along the token axis) on the GPU
against the oracle run sequence by sequence."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
import oracle
import momentum_delta_rule_mdn_b200 as mdn
from momentum_delta_rule_mdn_b200 import _lib
from parity import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu

GATES = ("alpha_log", "mu_log", "beta", "eta")


def _packed(lens, H, d, dtype, seed, state_std=0.05):
    """Packed inputs for the given lengths: (host Inputs of one batch row, device
    dict of [total,H,...] tensors, cu_seqlens (numpy, device), S0, M0 [N,H,d,d])."""
    total = int(sum(lens))
    spec = mi.Spec("varlen", B=1, T=total, H=H, d=d, dtype=dtype, seed=seed)
    inp = mi.make_inputs(spec)
    st = mi.make_inputs(mi.Spec("varlen_states", B=len(lens), T=0, H=H, d=d,
                                state_std=state_std, seed=seed + 1))
    dev = {k: v[0] for k, v in mi.to_torch(inp, "cuda").items() if v is not None}
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_dev = torch.from_numpy(cu).cuda()
    S0 = torch.from_numpy(st.S0).cuda() if st.S0 is not None else None
    M0 = torch.from_numpy(st.M0).cuda() if st.M0 is not None else None
    return inp, dev, cu, cu_dev, st.S0, st.M0, S0, M0


def _ref(inp, cu, S0, M0):
    f = lambda x: x[0]
    return oracle.chunk_fwd_varlen(f(inp.q), f(inp.k), f(inp.v), f(inp.alpha_log),
                                   f(inp.mu_log), f(inp.beta), f(inp.eta), cu, inp.d_corr,
                                   S0, M0)


@pytest.mark.parametrize("dtype,d,flags", [
    ("bf16", 128, 0),                        # tensor-core path
    ("bf16", 128, _lib.MDN_FORCE_SIMT),      # CUDA-core path, bf16 storage
    ("f32", 64, 0),
    ("f32", 128, 0),
])
def test_varlen_matches_oracle(dtype, d, flags):
    """Lengths around the chunk size, empty sequences among them."""
    lens = [0, 1, 63, 64, 65, 200, 0, 130, 7]
    H = 3
    inp, dev, cu, cu_dev, S0n, M0n, S0, M0 = _packed(lens, H, d, dtype, seed=401)
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(*(dev[k] for k in ("q", "k", "v")),
                                           *(dev[g] for g in GATES), cu_dev, inp.d_corr,
                                           S0, M0, flags=flags | _lib.MDN_CHECK_FINITE)
    torch.cuda.synchronize()
    ro, rvt, rS, rM = _ref(inp, cu, S0n, M0n)
    tol = TOL[dtype]
    for name, g, r in (("o", o, ro), ("vtilde", vt, rvt), ("S_T", S_T, rS), ("M_T", M_T, rM)):
        e = rel_l2(to_np(g), r)
        assert e <= tol, (name, e)
    # per sequence as well, so that a short sequence cannot hide in the total
    o_np, vt_np = to_np(o), to_np(vt)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        if b > a:
            assert rel_l2(o_np[a:b], ro[a:b]) <= tol, ("o", s)
            assert rel_l2(vt_np[a:b], rvt[a:b]) <= tol, ("vtilde", s)
        assert rel_l2(to_np(S_T[s]), rS[s]) <= tol, ("S_T", s)
    for s in (0, 6):  # empty sequences: the entering states pass through exactly
        assert torch.equal(S_T[s], S0[s]) and torch.equal(M_T[s], M0[s])


def test_varlen_equal_lengths_equal_the_batched_pass():
    """N sequences of one length (a multiple of the chunk) packed: bit-identical
    to mdn_chunk_fwd with B = N (same chunks, same chains, same arithmetic)."""
    N, L, H, d = 3, 256, 4, 128
    spec = mi.Spec("varlen_eq", B=N, T=L, H=H, d=d, state_std=0.02, seed=402)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    ref = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in GATES), inp.d_corr,
                        dev["S0"], dev["M0"])
    flat = lambda t: t.reshape((N * L,) + tuple(t.shape[2:])).contiguous()
    cu = torch.arange(N + 1, dtype=torch.int32, device="cuda") * L
    got = mdn.chunk_fwd_varlen(*(flat(dev[k]) for k in ("q", "k", "v")),
                               *(flat(dev[g]) for g in GATES), cu, inp.d_corr,
                               dev["S0"], dev["M0"])
    torch.cuda.synchronize()
    assert torch.equal(got[0], flat(ref[0])) and torch.equal(got[1], flat(ref[1]))
    assert torch.equal(got[2], ref[2]) and torch.equal(got[3], ref[3])


def test_varlen_layer_budget_length_mix():
    """The layer workload's token budget (8192 tokens, H = 8, d = 128, bf16) as a
    mix of nine sequence lengths, against the oracle on every head."""
    lens = [3000, 1500, 64, 2500, 1, 700, 300, 127, 0]
    lens[-1] = 8192 - sum(lens[:-1])
    inp, dev, cu, cu_dev, S0n, M0n, S0, M0 = _packed(lens, 8, 128, "bf16", seed=403,
                                                     state_std=0.01)
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(*(dev[k] for k in ("q", "k", "v")),
                                           *(dev[g] for g in GATES), cu_dev, inp.d_corr,
                                           S0, M0)
    torch.cuda.synchronize()
    ro, rvt, rS, rM = _ref(inp, cu, S0n, M0n)
    for name, g, r in (("o", o, ro), ("vtilde", vt, rvt), ("S_T", S_T, rS), ("M_T", M_T, rM)):
        assert rel_l2(to_np(g), r) <= TOL["bf16"], name


def test_varlen_many_sequences_beyond_the_rank_limit():
    """More sequences (2,100) than the setup ranks by length (2,048): the work
    order falls back to the call order; lengths 0..150 at random, H = 1,
    bf16, d = 128, against the oracle over the whole batch and per sequence."""
    rng = np.random.default_rng(405)
    lens = [int(x) for x in rng.integers(0, 151, size=2100)]
    inp, dev, cu, cu_dev, S0n, M0n, S0, M0 = _packed(lens, 1, 128, "bf16", seed=406,
                                                     state_std=0.01)
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(*(dev[k] for k in ("q", "k", "v")),
                                           *(dev[g] for g in GATES), cu_dev, inp.d_corr,
                                           S0, M0, flags=_lib.MDN_CHECK_FINITE)
    torch.cuda.synchronize()
    ro, rvt, rS, rM = _ref(inp, cu, S0n, M0n)
    for name, g, r in (("o", o, ro), ("vtilde", vt, rvt), ("S_T", S_T, rS), ("M_T", M_T, rM)):
        assert rel_l2(to_np(g), r) <= TOL["bf16"], name
    S_np = to_np(S_T)
    worst = max(rel_l2(S_np[s], rS[s]) for s in range(len(lens)) if lens[s] > 0)
    assert worst <= TOL["bf16"], worst


def test_varlen_longest_sequence_last_and_first():
    """The work order ranks the sequences by length (chains and chunks of the
    longest first): a call with the longest sequence last and one with it
    first both match the oracle."""
    lens = [130, 64, 1, 700, 65, 2000]
    outs = []
    for order in (lens, lens[::-1]):
        inp, dev, cu, cu_dev, S0n, M0n, S0, M0 = _packed(order, 2, 128, "bf16", seed=407,
                                                         state_std=0.02)
        o, vt, S_T, M_T = mdn.chunk_fwd_varlen(*(dev[k] for k in ("q", "k", "v")),
                                               *(dev[g] for g in GATES), cu_dev, inp.d_corr,
                                               S0, M0)
        torch.cuda.synchronize()
        ro, rvt, rS, rM = _ref(inp, cu, S0n, M0n)
        for name, g, r in (("o", o, ro), ("vtilde", vt, rvt), ("S_T", S_T, rS), ("M_T", M_T, rM)):
            assert rel_l2(to_np(g), r) <= TOL["bf16"], (name, order)


@pytest.mark.parametrize("cu_list,total", [
    ([0, 100, 50, 200], 200),   # decreasing
    ([0, 100, 150], 200),       # does not end at total_T
    ([5, 100, 200], 200),       # does not start at 0
])
def test_varlen_rejects_bad_offsets(cu_list, total):
    """A cu_seqlens that breaks the rules makes every sequence empty (in-bounds,
    S_T = S0) and is reported under MDN_CHECK_FINITE."""
    H, d, N = 2, 64, len(cu_list) - 1
    g = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = (torch.randn(total, H, d, device="cuda", generator=g) for _ in range(3))
    gates = [torch.full((total, H), x, device="cuda") for x in (-0.1, -0.2, 0.5, 1.0)]
    cu = torch.tensor(cu_list, dtype=torch.int32, device="cuda")
    S0 = torch.randn(N, H, d, d, device="cuda", generator=g)
    M0 = torch.randn(N, H, d, d, device="cuda", generator=g)
    with pytest.raises(mdn.MDNError, match="INVALID_ARG"):
        mdn.chunk_fwd_varlen(q, k, v, *gates, cu, 0.5, S0, M0, flags=_lib.MDN_CHECK_FINITE)
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(q, k, v, *gates, cu, 0.5, S0, M0)
    torch.cuda.synchronize()
    assert torch.equal(S_T, S0) and torch.equal(M_T, M0)


def test_varlen_all_empty_and_no_sequences():
    H, d = 2, 128
    S0 = torch.randn(3, H, d, d, device="cuda")
    M0 = torch.randn(3, H, d, d, device="cuda")
    e = lambda *s, dt=torch.bfloat16: torch.empty(s, dtype=dt, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(e(0, H, d), e(0, H, d), e(0, H, d),
                                           *(e(0, H, dt=torch.float32) for _ in range(4)),
                                           cu, 0.5, S0, M0, flags=_lib.MDN_CHECK_FINITE)
    assert torch.equal(S_T, S0) and torch.equal(M_T, M0)
    cu1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, vt, S_T, M_T = mdn.chunk_fwd_varlen(e(0, H, d), e(0, H, d), e(0, H, d),
                                           *(e(0, H, dt=torch.float32) for _ in range(4)),
                                           cu1, 0.5)
    assert S_T.shape == (0, H, d, d)
