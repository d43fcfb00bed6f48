"""Per-phase cycle counts of the backward pass's per-chunk kernels and of its
reverse chain, from a diagnostic build of the library.

    python -m momentum_delta_rule_mdn_b200.bwd_phase_clocks [WORKLOAD]

Compiles chunk_bwd_tc.cu and chunk_bwd_chain_tc.cu with MDN_PHASE_CLOCKS (the
phase counters are compiled out of the normal build) into a separate library
under _build/diag, runs mdn_chunk_bwd on the synthetic workload (default 1,
the 400M-layer shape) from the forward pass's vtilde, and prints, per kernel,
the cycles between its barriers as thread 0 of every CTA sees them (averaged
over CTAs), and for the reverse chain the laps of CTA 0's MMA lane, TMA lane
and one Y-row chain warp per chunk.  Nothing is checked (the tests do that).
"""
from __future__ import annotations

import ctypes
import glob
import os
import subprocess
import sys

import torch

import mdn_inputs as mi

from . import _lib, api, build_lib

DIAG = os.path.join(build_lib.BUILD, "diag")

# lap names, in the order of the kernels' counters
STATE = ["copies_issue+sync", "copy_wait+inner_products", "mma_wait", "dY_rows_epilogue",
         "dO_rows_epilogue+sums", "record+dealloc"]
LOCAL = ["gates+sync", "tma_wait", "stage1_mma+Gamma", "stage1_epilogue", "stage2_wait",
         "stage2_dY_rows", "dq_dk_staging", "coeff_0", "coeff_scans", "coeff_row_col_sums",
         "coeff_R", "coeff_U", "coeff_cumsums", "coeff_stores"]
PREP = ["gates+sync", "staging", "mma1_wait", "U_P_epilogue+mma2", "D_stores"]
CHAIN_MMA = ["loop", "wait_state", "issue_A1_EF", "wait_T_U", "wait_Y", "issue_A2", "issue_A3",
             "wait_next_KQ_slot"]
CHAIN_TMA = ["wait_KQ_slot", "wait_slice_slot", "wait_T_U_slot"]
CHAIN_Y = ["wait_slices", "wait_A1", "Y", "Y_handoff", "wait_A2", "state", "state_handoff",
           "adjoint_image_stores"]


def build_diag() -> str:
    build_lib.build()
    os.makedirs(DIAG, exist_ok=True)
    flags = build_lib.NVCC_FLAGS + ["-DMDN_PHASE_CLOCKS"]
    csrc = os.path.join(build_lib.PKG, "csrc")
    objs = []
    for name in ("chunk_bwd_tc", "chunk_bwd_chain_tc"):
        obj = os.path.join(DIAG, name + ".o")
        subprocess.run([build_lib.nvcc()] + flags + ["-c", os.path.join(csrc, name + ".cu"), "-o", obj],
                       check=True)
        objs.append(obj)
    keep = [o for o in glob.glob(os.path.join(build_lib.BUILD, "*.o"))
            if os.path.basename(o) not in ("chunk_bwd_tc.o", "chunk_bwd_chain_tc.o")]
    so = os.path.join(DIAG, "libmdn_phase_clocks.so")
    subprocess.run([build_lib.nvcc()] + build_lib.ARCH + ["-shared", "-o", so] + keep + objs,
                   check=True)
    return so


def main(argv) -> None:
    spec = mi.WORKLOADS[int(argv[0]) if argv else 1]
    torch.cuda.set_device(0)
    lib = _lib.load(build_diag())
    api._handle = lib  # every call below goes to the diagnostic build
    lib.mdn_diag_bwd_clock.argtypes = [ctypes.c_void_p]
    lib.mdn_diag_chain_clock.argtypes = [ctypes.c_void_p]
    inp = mi.make_inputs(spec)
    dev = mi.to_torch(inp, "cuda")
    gates = ("alpha_log", "mu_log", "beta", "eta")
    o, vt, _, _ = api.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), inp.d_corr)
    do = torch.randn(o.shape, generator=torch.Generator().manual_seed(3)).to(o)

    def call():
        api.chunk_bwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), inp.d_corr, vt, do)

    call()
    torch.cuda.synchronize()
    buf = torch.zeros(3 * 32, device="cuda")
    lib.mdn_diag_bwd_clock(ctypes.c_void_p(buf.data_ptr()))
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    lib.mdn_diag_bwd_clock(None)
    cbuf = torch.zeros(64, device="cuda")
    lib.mdn_diag_chain_clock(ctypes.c_void_p(cbuf.data_ptr()))
    call()
    torch.cuda.synchronize()
    lib.mdn_diag_chain_clock(None)
    c = buf.cpu().numpy().reshape(3, 32)
    print(f"{spec.name}: cycles per CTA (thread 0, averaged over CTAs)")
    for k, (name, laps) in enumerate((("state products", STATE), ("local products", LOCAL),
                                      ("chain operands", PREP))):
        n = max(float(c[k, 31]), 1.0)
        per = {lap: round(float(c[k, i]) / n) for i, lap in enumerate(laps)}
        print(f"  {name}: {per} sum {round(float(c[k, :31].sum()) / n)}")
    nt = (spec.T + 63) // 64
    cc = cbuf.cpu().numpy()
    print(f"reverse chain, CTA 0, cycles per chunk ({nt} chunks)")
    for base, name, laps in ((0, "MMA lane", CHAIN_MMA), (20, "TMA lane", CHAIN_TMA),
                             (40, "Y-row chain warp", CHAIN_Y)):
        per = {lap: round(float(cc[base + i]) / nt) for i, lap in enumerate(laps)}
        print(f"  {name}: {per} sum {round(float(cc[base:base + 20].sum()) / nt)}")


if __name__ == "__main__":
    main(sys.argv[1:])
