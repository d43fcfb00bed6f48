"""Run one of the library's kernels on a synthetic workload a few times, for an
external profiler (ncu) to capture: a fixed, small command per kernel.

    python -m momentum_delta_rule_mdn_b200.profile_cases CASE [WORKLOAD] [REPS]

CASE      chunk      mdn_chunk_fwd over the workload's batch (both chunk kernels)
          preact     mdn_chunk_fwd_preact (gates from pre-activations) over the batch
          step       one mdn_step token for every head of the decode workload
                     (B=256, H=16, d=128: S and M are 2 x 268 MB, far above L2)
          gate_prep  mdn_chunk_gate_prep (la, lm, lc, b and Gamma) on the workload's gates
          gates      mdn_gate_params on the workload's pre-activations
          bwd        mdn_chunk_bwd over the batch, from the forward pass's vtilde and a
                     seeded cotangent of o (every backward kernel)
WORKLOAD  index or name of a synthetic workload (default 2, the 1.3B-layer shape)
REPS      calls (default 3)

Inputs come from the seeded generator; nothing is checked (the tests do that).
"""
from __future__ import annotations

import sys

import torch

import mdn_inputs as mi

from . import api


def _spec(w: str) -> mi.Spec:
    if w.isdigit():
        return mi.WORKLOADS[int(w)]
    for s in mi.WORKLOADS:
        if s.name == w:
            return s
    raise SystemExit(f"unknown workload {w!r}")


def main(argv) -> None:
    case = argv[0] if argv else "chunk"
    spec = _spec(argv[1] if len(argv) > 1 else "2")
    reps = int(argv[2]) if len(argv) > 2 else 3
    torch.cuda.set_device(0)
    gates = ("alpha_log", "mu_log", "beta", "eta")
    if case == "step":
        dec = mi.WORKLOADS[4]
        tok = mi.make_inputs(mi.replace(dec, T=1, seed=dec.seed + 11))
        t = {k: v[:, 0].contiguous() for k, v in mi.to_torch(tok, "cuda").items() if v is not None}
        S = torch.randn((dec.B, dec.H, dec.d, dec.d), device="cuda") * 0.01
        M = torch.randn_like(S) * 0.01
        for _ in range(reps):
            api.step(t["q"], t["k"], t["v"], *(t[g] for g in gates), dec.q_corr, S, M,
                     want_vtilde=False)
    else:
        inp = mi.make_inputs(spec)
        dev = mi.to_torch(inp, "cuda")
        pre = [torch.from_numpy(p).cuda() for p in (inp.x_eta, inp.a_pre, inp.b_pre, inp.c_pre)]
        if case == "bwd":
            o, vt, _, _ = api.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates),
                                        inp.d_corr)
            do = torch.randn(o.shape, generator=torch.Generator().manual_seed(3)).to(o)
        for _ in range(reps):
            if case == "bwd":
                api.chunk_bwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), inp.d_corr,
                              vt, do)
            elif case == "chunk":
                api.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), inp.d_corr,
                              dev["S0"], dev["M0"])
            elif case == "preact":
                api.chunk_fwd_preact(dev["q"], dev["k"], dev["v"], *pre, s=spec.eta_scale,
                                     mu_log_min=spec.mu_log_min, d=inp.d_corr, S0=dev["S0"],
                                     M0=dev["M0"])
            elif case == "gate_prep":
                api.chunk_gate_prep(*(dev[g] for g in gates))
            elif case == "gates":
                api.gate_params(*pre, s=spec.eta_scale, mu_log_min=spec.mu_log_min)
            else:
                raise SystemExit(f"unknown case {case!r}")
    torch.cuda.synchronize()
    print(f"{case} on {spec.name if case != 'step' else mi.WORKLOADS[4].name}: {reps} call(s) ok")


if __name__ == "__main__":
    main(sys.argv[1:])
