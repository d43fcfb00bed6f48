"""The C ABI without a GPU: the library loads, exports every function that
include/*.h declares, and its host-side validation rejects bad arguments
before touching the device."""
import glob
import os
import re
import subprocess

import pytest

from momentum_delta_rule_mdn_b200 import _lib, build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return _lib.load()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(mdn_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("mdn_chunk_fwd", "mdn_step", "mdn_chunk_fwd_workspace_size", "mdn_status_string",
              "mdn_chunk_gate_prep", "mdn_abi_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mdn_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(_lib.SIGNATURES) <= exported


def test_status_strings(lib):
    assert lib.mdn_abi_version() == 1
    for s in range(6):
        assert lib.mdn_status_string(s).decode().startswith("MDN_")
    assert b"unknown" in lib.mdn_status_string(99)


def test_workspace_size_rules(lib):
    ws = lib.mdn_chunk_fwd_workspace_size
    assert ws(8, 4096, 16, 128, 128, 64, _lib.MDN_BF16) > 0
    assert ws(1, 0, 1, 64, 64, 64, _lib.MDN_F32) > 0
    assert ws(1, 256, 1, 96, 96, 64, _lib.MDN_F32) == 0      # unsupported d
    assert ws(1, 256, 1, 64, 128, 64, _lib.MDN_F32) == 0     # d_k != d_v
    assert ws(1, 256, 1, 64, 64, 32, _lib.MDN_F32) == 0      # unsupported C
    assert ws(-1, 256, 1, 64, 64, 64, _lib.MDN_F32) == 0
    assert ws(1, 256, 1, 64, 64, 64, 7) == 0                 # unknown dtype
    # grows with T and covers whole chunks of a ragged tail
    assert ws(1, 65, 1, 64, 64, 64, 0) == ws(1, 128, 1, 64, 64, 64, 0)
    assert ws(1, 129, 1, 64, 64, 64, 0) > ws(1, 128, 1, 64, 64, 64, 0)


def test_workspace_sized_by_path(lib):
    """The scratch holds only the regions of the path that runs: the tensor-core
    path (bf16, d = 128) its bf16 chunk operands and coefficient records, the
    CUDA-core path its fp32 coefficients, Gamma and U/Y/Z/O_inter."""
    wsf = lib.mdn_chunk_fwd_workspace_size_flags
    E = _lib
    MiB = 1 << 20
    for (B, T, H) in ((4, 2048, 8), (8, 4096, 16), (1, 16384, 16), (2, 200, 3)):
        chunks = B * H * ((T + 63) // 64)
        rows = chunks * 64
        up = lambda x: (x + 255) // 256 * 256
        tc = up(64 + (chunks + 1) * 4) + up(rows * 128 * 2) + up(rows * 128 * 2) \
            + up(rows * 256 * 2) + up(rows * 16)
        assert wsf(B, T, H, 128, 128, 64, E.MDN_BF16, 0) == tc
        assert lib.mdn_chunk_fwd_workspace_size(B, T, H, 128, 128, 64, E.MDN_BF16) == tc
        simt = up(64 + (chunks + 1) * 4) + 4 * up(rows * 4) + up(rows * 64 * 4) \
            + 4 * up(rows * 128 * 4)
        assert wsf(B, T, H, 128, 128, 64, E.MDN_BF16, E.MDN_FORCE_SIMT) == simt
        assert wsf(B, T, H, 128, 128, 64, E.MDN_F32, 0) == simt      # fp32 runs on CUDA cores
    assert wsf(4, 2048, 8, 128, 128, 64, E.MDN_BF16, 0) <= 70 * MiB
    assert wsf(8, 4096, 16, 128, 128, 64, E.MDN_BF16, 0) <= 0.6 * 1024 * MiB
    # d = 64 has no tensor-core path: the flag changes nothing
    assert wsf(1, 256, 2, 64, 64, 64, E.MDN_BF16, 0) == \
        wsf(1, 256, 2, 64, 64, 64, E.MDN_BF16, E.MDN_FORCE_SIMT)
    vws = lib.mdn_chunk_fwd_varlen_workspace_size_flags
    assert vws(3, 1000, 4, 128, 128, 64, E.MDN_BF16, 0) < \
        vws(3, 1000, 4, 128, 128, 64, E.MDN_BF16, E.MDN_FORCE_SIMT)
    assert lib.mdn_chunk_fwd_varlen_workspace_size(3, 1000, 4, 128, 128, 64, E.MDN_BF16) == \
        vws(3, 1000, 4, 128, 128, 64, E.MDN_BF16, 0)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_too_small_workspace_for_the_requested_path(lib):
    """A workspace sized for the default (tensor-core) path is rejected before any
    device work when MDN_FORCE_SIMT asks for the CUDA-core path."""
    E = _lib
    need_tc = lib.mdn_chunk_fwd_workspace_size_flags(1, 128, 1, 128, 128, 64, E.MDN_BF16, 0)
    need_simt = lib.mdn_chunk_fwd_workspace_size_flags(1, 128, 1, 128, 128, 64, E.MDN_BF16,
                                                       E.MDN_FORCE_SIMT)
    assert need_simt > need_tc
    assert _chunk(lib, dk=128, dv=128, wsb=need_tc, flags=E.MDN_FORCE_SIMT) == \
        E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, dk=128, dv=128, wsb=need_tc - 1) == E.MDN_ERR_INVALID_ARG


def test_status_query_validation(lib):
    assert lib.mdn_chunk_fwd_status(None, None) == _lib.MDN_ERR_INVALID_ARG
    assert lib.mdn_chunk_fwd_status(FAKE + 16, None) == _lib.MDN_ERR_INVALID_ARG


def test_noalloc_validates_before_any_device_work(lib):
    """Invalid or unsupported sizes get mdn_chunk_fwd's own errors without the
    library touching a device (this machine may have none: a device call would
    come back as MDN_ERR_CUDA); sizes beyond the fixed scratch are refused."""
    E = _lib

    def na(B=1, T=128, H=1, d=128, C=64, dt=E.MDN_BF16, flags=0, q=FAKE):
        return lib.mdn_chunk_fwd_noalloc(q, FAKE, FAKE, dt, FAKE, FAKE, FAKE, FAKE, 0.5, None,
                                         None, B, T, H, d, d, C, FAKE, FAKE, FAKE, FAKE, flags,
                                         None)
    assert na(d=96) == E.MDN_ERR_UNSUPPORTED
    assert na(C=32) == E.MDN_ERR_UNSUPPORTED
    assert na(dt=7) == E.MDN_ERR_UNSUPPORTED
    assert na(B=-1) == E.MDN_ERR_INVALID_ARG
    assert na(T=-5) == E.MDN_ERR_INVALID_ARG
    assert na(B=0) == E.MDN_OK
    assert na(B=8, T=4096, H=16) == E.MDN_ERR_UNSUPPORTED              # beyond 64 MiB


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=_lib.MDN_BF16, al=FAKE, ml=FAKE, be=FAKE, et=FAKE,
             d=0.5, S0=None, M0=None, B=1, T=128, H=1, dk=64, dv=64, C=64, o=FAKE, vt=FAKE,
             ST=FAKE, MT=FAKE, ws=FAKE, wsb=0, flags=0)
    a.update(kw)
    return lib.mdn_chunk_fwd(a["q"], a["k"], a["v"], a["dt"], a["al"], a["ml"], a["be"],
                             a["et"], a["d"], a["S0"], a["M0"], a["B"], a["T"], a["H"],
                             a["dk"], a["dv"], a["C"], a["o"], a["vt"], a["ST"], a["MT"],
                             a["ws"], a["wsb"], a["flags"], None)


def test_chunk_fwd_validation(lib):
    E = _lib
    assert _chunk(lib, dk=96, dv=96) == E.MDN_ERR_UNSUPPORTED
    assert _chunk(lib, C=32) == E.MDN_ERR_UNSUPPORTED
    assert _chunk(lib, dt=5) == E.MDN_ERR_UNSUPPORTED
    assert _chunk(lib, B=-1) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, C=0) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, flags=0x100) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, flags=_lib.MDN_SLICE32 | _lib.MDN_SLICE64) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, flags=_lib.MDN_SLICE64 | _lib.MDN_SLICE128) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, flags=_lib.MDN_SLICE32 | _lib.MDN_SLICE128) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, q=None) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, vt=None) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, ST=None) == E.MDN_ERR_INVALID_ARG
    assert _chunk(lib, k=FAKE + 4) == E.MDN_ERR_INVALID_ARG           # unaligned
    assert _chunk(lib, al=FAKE + 2) == E.MDN_ERR_INVALID_ARG          # gate not 4-byte aligned
    assert _chunk(lib, ws=FAKE + 16) == E.MDN_ERR_INVALID_ARG         # workspace not 256-aligned
    need = lib.mdn_chunk_fwd_workspace_size(1, 128, 1, 64, 64, 64, _lib.MDN_BF16)
    assert _chunk(lib, wsb=need - 1) == E.MDN_ERR_INVALID_ARG         # workspace too small
    assert _chunk(lib, B=0) == E.MDN_OK                               # nothing to do
    assert _chunk(lib, H=0, q=None) == E.MDN_OK


def test_step_and_gate_prep_validation(lib):
    E = _lib
    st = lambda **kw: lib.mdn_step(kw.get("q", FAKE), FAKE, FAKE, kw.get("dt", 1), FAKE, FAKE,
                                   FAKE, FAKE, 0.5, kw.get("S", FAKE), FAKE, kw.get("B", 2), 3,
                                   kw.get("d", 128), kw.get("d", 128), FAKE, None,
                                   kw.get("flags", 0), None)
    assert st(d=32) == E.MDN_ERR_UNSUPPORTED
    assert st(q=None) == E.MDN_ERR_INVALID_ARG
    assert st(S=FAKE + 8) == E.MDN_ERR_INVALID_ARG
    assert st(q=FAKE + 1) == E.MDN_ERR_INVALID_ARG                   # bf16 needs 2-byte alignment
    assert st(flags=1) == E.MDN_ERR_INVALID_ARG
    assert st(B=0) == E.MDN_OK
    gp = lambda **kw: lib.mdn_chunk_gate_prep(FAKE, FAKE, FAKE, FAKE, 1, kw.get("T", 100), 1,
                                              kw.get("C", 64), kw.get("la", FAKE), FAKE, FAKE,
                                              FAKE, None, None)
    assert gp(C=16) == E.MDN_ERR_UNSUPPORTED
    assert gp(la=None) == E.MDN_ERR_INVALID_ARG
    assert gp(T=0) == E.MDN_OK


def test_gate_params_and_delta_norm_validation(lib):
    E = _lib
    inf = float("inf")

    def gp(n=10, s=1.0, mn=-2.0, act=E.MDN_ETA_TANH, x=FAKE, out=FAKE):
        return lib.mdn_gate_params(x, FAKE, FAKE, FAKE, n, s, mn, act, out, FAKE, FAKE, FAKE,
                                   None)
    assert gp(n=-1) == E.MDN_ERR_INVALID_ARG
    assert gp(act=2) == E.MDN_ERR_INVALID_ARG
    assert gp(s=inf) == E.MDN_ERR_INVALID_ARG
    assert gp(mn=float("nan")) == E.MDN_ERR_INVALID_ARG
    assert gp(x=None) == E.MDN_ERR_INVALID_ARG
    assert gp(out=FAKE + 2) == E.MDN_ERR_INVALID_ARG                 # not 4-byte aligned
    assert gp(n=0) == E.MDN_OK
    assert gp(n=0, act=E.MDN_ETA_2SIGMOID, x=None) == E.MDN_OK       # nothing to read

    def dn(B=2, ds=FAKE, d=128):
        return lib.mdn_step_delta_norm(FAKE, FAKE, FAKE, E.MDN_BF16, FAKE, FAKE, FAKE, FAKE, 0.5,
                                       FAKE, FAKE, B, 3, d, d, FAKE, None, ds, 0, None)
    assert dn(ds=None) == E.MDN_ERR_INVALID_ARG
    assert dn(ds=FAKE + 1) == E.MDN_ERR_INVALID_ARG
    assert dn(d=32) == E.MDN_ERR_UNSUPPORTED
    assert dn(B=0, ds=None) == E.MDN_OK


def test_varlen_workspace_and_validation(lib):
    E = _lib
    ws = lib.mdn_chunk_fwd_varlen_workspace_size
    assert ws(4, 8192, 8, 128, 128, 64, E.MDN_BF16) > 0
    assert ws(0, 0, 8, 128, 128, 64, E.MDN_BF16) > 0
    assert ws(-1, 100, 8, 128, 128, 64, E.MDN_BF16) == 0
    assert ws(2, -5, 8, 128, 128, 64, E.MDN_BF16) == 0
    assert ws(2, 100, 8, 96, 96, 64, E.MDN_BF16) == 0                  # unsupported d
    # room for the worst split: every sequence ends one token into a chunk
    assert ws(5, 640, 1, 64, 64, 64, E.MDN_F32) == ws(10, 320, 1, 64, 64, 64, E.MDN_F32)
    assert ws(5, 641, 1, 64, 64, 64, E.MDN_F32) == ws(5, 640, 1, 64, 64, 64, E.MDN_F32)
    need = ws(2, 100, 1, 64, 64, 64, E.MDN_F32)

    def vl(N=2, total=100, cu=FAKE, wsb=need, flags=0, q=FAKE, S_T=FAKE):
        return lib.mdn_chunk_fwd_varlen(q, FAKE, FAKE, E.MDN_F32, FAKE, FAKE, FAKE, FAKE, 0.5,
                                        cu, N, total, None, None, 1, 64, 64, 64, FAKE, FAKE,
                                        S_T, FAKE, FAKE, wsb, flags, None)
    assert vl(cu=None) == E.MDN_ERR_INVALID_ARG
    assert vl(cu=FAKE + 2) == E.MDN_ERR_INVALID_ARG
    assert vl(q=None) == E.MDN_ERR_INVALID_ARG
    assert vl(S_T=FAKE + 4) == E.MDN_ERR_INVALID_ARG
    assert vl(wsb=need - 1) == E.MDN_ERR_INVALID_ARG
    assert vl(flags=E.MDN_TEST_NO_INTRA) == E.MDN_ERR_INVALID_ARG
    assert vl(N=-1) == E.MDN_ERR_INVALID_ARG
    assert vl(N=0, cu=None) == E.MDN_OK


def test_bwd_workspace_and_validation(lib):
    E = _lib
    ws = lib.mdn_chunk_bwd_workspace_size
    assert ws(4, 2048, 8, 128, 128, 64, E.MDN_BF16) > 0
    assert ws(4, 2048, 8, 96, 96, 64, E.MDN_BF16) == 0
    assert ws(1, 65, 1, 64, 64, 64, E.MDN_F32) == ws(1, 128, 1, 64, 64, 64, E.MDN_F32)
    need = ws(1, 100, 1, 64, 64, 64, E.MDN_F32)

    def bw(T=100, flags=0, wsb=need, dq=FAKE, vt=FAKE, dS0=FAKE, dST=None, gate=FAKE):
        return lib.mdn_chunk_bwd(FAKE, FAKE, FAKE, E.MDN_F32, gate, FAKE, FAKE, FAKE, 0.5, None,
                                 None, vt, FAKE, dST, None, 1, T, 1, 64, 64, 64, dq, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, FAKE, dS0, FAKE, FAKE, wsb, flags, None)
    assert bw(flags=4) == E.MDN_ERR_INVALID_ARG
    assert bw(vt=None) == E.MDN_ERR_INVALID_ARG
    assert bw(dq=FAKE + 4) == E.MDN_ERR_INVALID_ARG
    assert bw(dS0=None) == E.MDN_ERR_INVALID_ARG
    assert bw(dST=FAKE + 8) == E.MDN_ERR_INVALID_ARG
    assert bw(gate=FAKE + 2) == E.MDN_ERR_INVALID_ARG
    assert bw(wsb=need - 1) == E.MDN_ERR_INVALID_ARG
    assert bw(T=-1) == E.MDN_ERR_INVALID_ARG


def test_preact_validation(lib):
    """The fused-gate pass validates its gate constants and pointers before any
    device work."""
    E = _lib
    inf = float("inf")

    def pa(act=E.MDN_ETA_TANH, s=1.0, mn=-2.0, x=FAKE, d=64, B=1):
        return lib.mdn_chunk_fwd_preact(FAKE, FAKE, FAKE, E.MDN_BF16, x, FAKE, FAKE, FAKE, s, mn,
                                        act, 0.5, None, None, B, 128, 1, d, d, 64, FAKE, FAKE,
                                        FAKE, FAKE, FAKE, 0, 0, None)
    assert pa(act=2) == E.MDN_ERR_INVALID_ARG
    assert pa(s=inf) == E.MDN_ERR_INVALID_ARG
    assert pa(mn=float("nan")) == E.MDN_ERR_INVALID_ARG
    assert pa(x=None) == E.MDN_ERR_INVALID_ARG
    assert pa(x=FAKE + 2) == E.MDN_ERR_INVALID_ARG
    assert pa(d=96) == E.MDN_ERR_UNSUPPORTED
    assert pa(B=0) == E.MDN_OK
