"""mdn_chunk_fwd_noalloc: the forward pass for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), called
through the C ABI and checked against mdn_chunk_fwd with a caller workspace.

Two calls in a row with different inputs and sizes: the array keeps the
previous call's contents, and the second result must not depend on them.
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import mdn_inputs as mi
import momentum_delta_rule_mdn_b200 as mdn
from momentum_delta_rule_mdn_b200 import _lib, build_lib
from parity import TOL, rel_l2, to_np

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return _lib.load()


def _noalloc(lib, dev, spec, d_corr):
    B, T, H, d = spec.B, spec.T, spec.H, spec.d
    o = torch.empty_like(dev["q"])
    vt = torch.empty_like(dev["q"])
    S_T = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    M_T = torch.empty_like(S_T)
    code = _lib.MDN_BF16 if dev["q"].dtype == torch.bfloat16 else _lib.MDN_F32
    p = lambda t: None if t is None else t.data_ptr()
    st = lib.mdn_chunk_fwd_noalloc(
        p(dev["q"]), p(dev["k"]), p(dev["v"]), code, p(dev["alpha_log"]), p(dev["mu_log"]),
        p(dev["beta"]), p(dev["eta"]), d_corr, p(dev["S0"]), p(dev["M0"]), B, T, H, d, d, 64,
        p(o), p(vt), p(S_T), p(M_T), 0, torch.cuda.current_stream().cuda_stream)
    assert st == _lib.MDN_OK, lib.mdn_status_string(st)
    return o, vt, S_T, M_T


def test_noalloc_matches_workspace_entry_point_twice(lib):
    specs = [mi.Spec("noalloc_a", B=2, T=320, H=4, d=128, state_std=0.01, seed=501),
             mi.Spec("noalloc_b", B=1, T=200, H=3, d=64, dtype="f32", seed=502)]
    for spec in specs:
        assert mdn.chunk_fwd_workspace_size(spec.B, spec.T, spec.H, spec.d) <= SCRATCH_BYTES
        inp = mi.make_inputs(spec)
        dev = mi.to_torch(inp, "cuda")
        got = _noalloc(lib, dev, spec, inp.d_corr)
        ref = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"],
                            dev["beta"], dev["eta"], inp.d_corr, dev["S0"], dev["M0"])
        torch.cuda.synchronize()
        tol = TOL[spec.dtype]
        for g, r in zip(got, ref):
            assert rel_l2(to_np(g), to_np(r)) <= tol
            assert np.all(np.isfinite(to_np(g)))


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    B, T, H, d = 8, 4096, 16, 128
    assert lib.mdn_chunk_fwd_workspace_size(B, T, H, d, d, 64, _lib.MDN_BF16) > SCRATCH_BYTES
    fake = 0x10000
    st = lib.mdn_chunk_fwd_noalloc(fake, fake, fake, _lib.MDN_BF16, fake, fake, fake, fake,
                                   0.5, None, None, B, T, H, d, d, 64, fake, fake, fake, fake,
                                   0, None)
    assert st == _lib.MDN_ERR_UNSUPPORTED


def test_noalloc_invalid_sizes_then_a_valid_call(lib):
    """Unsupported d or C and a negative size get mdn_chunk_fwd's own errors
    through the no-allocation entry point; a valid call right after is still
    correct."""
    fake = 0x10000
    bad = lambda d, C, B=1: lib.mdn_chunk_fwd_noalloc(
        fake, fake, fake, _lib.MDN_BF16, fake, fake, fake, fake, 0.5, None, None, B, 128, 2,
        d, d, C, fake, fake, fake, fake, 0, None)
    assert bad(96, 64) == _lib.MDN_ERR_UNSUPPORTED
    assert bad(128, 32) == _lib.MDN_ERR_UNSUPPORTED
    assert bad(128, 64, B=-1) == _lib.MDN_ERR_INVALID_ARG
    spec = mi.Spec("noalloc_c", B=1, T=130, H=2, d=128, state_std=0.01, seed=503)
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    got = _noalloc(lib, dev, spec, inp.d_corr)
    ref = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["alpha_log"], dev["mu_log"],
                        dev["beta"], dev["eta"], inp.d_corr, dev["S0"], dev["M0"])
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert rel_l2(to_np(g), to_np(r)) <= TOL["bf16"]
