"""Benchmark of the MDN hot path: one step = mdn_chunk_fwd over one batch of the
workload plus one mdn_step decode token continuing from the pass's (S_T, M_T).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME|INDEX]

Prints ONE JSON line on rank 0.  For N > 1 launch with torch.distributed.run:
each rank processes its own independently seeded batch (heads are independent,
so there is no collective on the data path); the step time is the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mdn_inputs as mi  # noqa: E402

METRIC = "MDN chunk-fwd tokens/s (d=128, bf16 in/fp32 state) and % tensor/HBM roofline"
DEFAULT_WORKLOAD = 2           # the largest single-GPU workload: B=8, H=16, T=4096, d=128, S0/M0 != 0
SIDE_WORKLOADS = (1, 3)        # timed the same way, reported beside the headline
L2_FLUSH_BYTES = 256 << 20     # > 126 MB of L2
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x FP32 lanes x FMA x max clock


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def load_traffic():
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            return json.load(f)
    except Exception:
        return {}


def pass_work(spec: mi.Spec):
    """The chunk pass's algorithmic minimum (the method's own contractions and
    the bytes it must move), per token-head: flops = 12 C d + 12 d^2 (the six
    C^2-type products K K^T, Qhat K^T, T V, T Y, T Z and the intra-chunk output,
    and the six C d^2-type products Y S, Z M, Qhat S, Qhat M and the two state
    increments; the T solve and Gamma excluded); bytes = q, k, v read and o,
    vtilde written in the input dtype, plus four fp32 gates; plus, per head, the
    fp32 S_T, M_T written and S0, M0 read when given.  Returns (bytes, flops)."""
    th = spec.B * spec.T * spec.H
    d, C = spec.d, spec.C
    elt = 2 if spec.dtype == "bf16" else 4
    heads = spec.B * spec.H
    states = 2 * heads * d * d * 4 * (2 if spec.state_std > 0 else 1)
    return th * (5 * d * elt + 16) + states, th * (12.0 * C * d + 12.0 * d * d)


def bwd_work(spec: mi.Spec, with_state_cot: bool = False):
    """The backward pass's algorithmic work per token-head, from its chunkwise
    form (per chunk of C tokens, d_k = d_v = d):
      C^2 d products: K K^T and Qhat K^T (T and Att rebuilt), Att^T dO, T^T dVtilde,
        dO Vt^T, dY Vt^T, Qhat K^T, K K^T (the chunk-local adjoints), [dOVG; dPK] K
        and [dOVG^T | dPKa^T] [Qhat; K]: 28 C^2 d flops
      C d^2 products: U = K^T [.. T^T] (counted as 4 C^2 d above), D = K^T [Gamma Vt |
        w Vt], K [dS | dM], U dVtilde, E and F, and the six state products dO S^T,
        dO M^T, dY S^T, dY M^T, Vt dS^T, Vt dM^T: 28 C d^2 flops
    so 28 C d + 28 d^2 flops per token-head (2.33 times the forward's); bytes =
    q, k, vtilde, d_o read in the input dtype and four fp32 gates read, dq, dk,
    dv and four gate gradients written in fp32; per head, dS0 and dM0 written
    and S0, M0 (and dS_T, dM_T when given) read in fp32.  Returns (bytes, flops)."""
    th = spec.B * spec.T * spec.H
    d, C = spec.d, spec.C
    elt = 2 if spec.dtype == "bf16" else 4
    heads = spec.B * spec.H
    n_state = 2 + (2 if spec.state_std > 0 else 0) + (2 if with_state_cot else 0)
    return (th * (4 * d * elt + 16 + 3 * d * 4 + 16) + heads * n_state * d * d * 4,
            th * (28.0 * C * d + 28.0 * d * d))


def token_bytes(spec: mi.Spec) -> int:
    """One decode token for every head: S and M read and written (fp32), q, k,
    v read, o written, four gates."""
    heads, d = spec.B * spec.H, spec.d
    elt = 2 if spec.dtype == "bf16" else 4
    return heads * (4 * d * d * 4 + 4 * d * elt + 16)


def kernel_work(name: str, spec: mi.Spec):
    """Algorithmic work of one launch of a kernel: (bound, amount, unit-of-peak).
    The tensor-core chunk kernels are charged the whole pass's algorithmic
    bytes (they split one pass between them; neither alone has a minimum of
    its own), the CUDA-core kernels their fp32 flops, the decode step its
    bytes."""
    th = spec.B * spec.T * spec.H          # token-heads
    d, C = spec.d, spec.C
    heads = spec.B * spec.H
    if name in ("inter_tc", "intra_tc"):
        return "hbm", pass_work(spec)[0], "GB/s"
    if name == "inter_simt":
        return "alu", th * 12.0 * d * d, "TFLOP/s"
    if name == "intra_simt":
        return "alu", th * 5.0 * C * d, "TFLOP/s"
    if name == "output_simt":
        return "alu", th * 4.0 * C * d, "TFLOP/s"
    if name == "gate_prep":
        return "hbm", th * (16 + 16 + 4 * C), "GB/s"
    if name == "step":
        return "hbm", heads * (4 * d * d * 4 + 3 * d * 2 + 16 + 2 * d * 2), "GB/s"
    return None, 0.0, ""


def fractions(nbytes: float, flops: float, sec: float, hbm: float, bf16: float) -> dict:
    """HBM, tensor and roofline fractions of work done in `sec` seconds:
    roofline = max(flops / tensor peak, bytes / HBM peak) / sec."""
    if sec <= 0:
        return {"hbm_frac": None, "tensor_frac": None, "roofline_frac": None}
    return {"achieved_gbs": round(nbytes / sec / 1e9, 1),
            "achieved_tflops": round(flops / sec / 1e12, 2),
            "hbm_frac": round(nbytes / sec / 1e9 / hbm, 4),
            "tensor_frac": round(flops / sec / 1e12 / bf16, 4),
            "roofline_frac": round(max(flops / (bf16 * 1e12), nbytes / (hbm * 1e9)) / sec, 4)}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clock record
            self.err = str(e)

    _NAMES = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
              0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
              0x100: "display_clock_setting", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self._NAMES.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "source": "nvml"}


# ---------------------------------------------------------------- our path
def decode_token(spec: mi.Spec, seed: int):
    """One decode token per (b, h): q, k, v [B,H,d] and gates [B,H] (stored dtypes)."""
    s = mi.replace(spec, T=1, seed=seed, state_std=0.0)
    inp = mi.make_inputs(s)
    return inp


class Pass:
    """One workload's step (mdn_chunk_fwd over the batch + one decode token that
    continues from its (S_T, M_T)) with its device buffers, ready to time."""

    def __init__(self, mdn, spec: mi.Spec, device):
        self.mdn, self.spec = mdn, spec
        self.inp = mi.make_inputs(spec)
        self.tok = decode_token(spec, spec.seed + 1)
        self.dev = mi.to_torch(self.inp, device)
        self.dtok = {k: (v[:, 0].contiguous() if v is not None else None)
                     for k, v in mi.to_torch(self.tok, device).items()}
        B, T, H, d = spec.B, spec.T, spec.H, spec.d
        self.ws = torch.empty(mdn.chunk_fwd_workspace_size(B, T, H, d, spec.C, self.dev["q"].dtype),
                              dtype=torch.uint8, device=device)
        self.out = (torch.empty_like(self.dev["q"]), torch.empty_like(self.dev["q"]),
                    torch.empty((B, H, d, d), dtype=torch.float32, device=device),
                    torch.empty((B, H, d, d), dtype=torch.float32, device=device))
        self.o1 = torch.empty_like(self.dtok["q"])

    def step(self):
        g = ("alpha_log", "mu_log", "beta", "eta")
        dev, dtok, spec = self.dev, self.dtok, self.spec
        self.mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[x] for x in g), self.inp.d_corr,
                           dev["S0"], dev["M0"], spec.C, out=self.out, workspace=self.ws)
        self.mdn.step(dtok["q"], dtok["k"], dtok["v"], *(dtok[x] for x in g), self.inp.d_corr,
                      self.out[2], self.out[3], o=self.o1, want_vtilde=False)

    def time(self, steps: int, warmup: int, flush, world: int, clock=None):
        """Per-step device times (ms) of `steps` steps after `warmup` untimed ones,
        L2 flushed (untimed) before each; then the library's per-kernel times
        from a second, untimed pass over the same number of steps (its events
        between kernels would otherwise serialise the two chunk kernels, which
        overlap in the timed pass)."""
        mdn = self.mdn
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            flush.zero_()
            self.step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        with (clock if clock is not None else _Null()):
            for i in range(steps):
                flush.zero_()
                ev[i][0].record(stream)
                self.step()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
        barrier(world)
        step_ms = [a.elapsed_time(b) for a, b in ev]
        mdn.profile_enable(True)
        mdn.profile_read(reset=True)
        for _ in range(steps):
            flush.zero_()
            self.step()
        torch.cuda.synchronize()
        kernels = mdn.profile_read(reset=True)
        mdn.profile_enable(False)
        status = mdn.chunk_fwd_status(self.ws)
        if status != 0:
            raise RuntimeError(f"chunk pass reported {mdn.status_string(status)}")
        return step_ms, kernels


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def pass_summary(spec: mi.Spec, ms: float, kernels: dict, steps: int, hbm: float, bf16: float):
    """Throughput and roofline fractions of one workload's step: over the whole
    step (pass + decode token) and over the pass's dominant kernel."""
    nbytes, flops = pass_work(spec)
    tb = token_bytes(spec)
    out = {"workload": spec.name, "ms_per_step": round(ms, 5),
           "tokens_per_s": round(spec.B * spec.T / (ms * 1e-3), 1),
           "step": fractions(nbytes + tb, flops, ms * 1e-3, hbm, bf16),
           "kernels_us": {k: round(v[0] / v[1] * 1e3, 2) for k, v in kernels.items()}}
    chunk = {k: v for k, v in kernels.items() if k != "step"}
    if chunk:
        name, (tot, n) = max(chunk.items(), key=lambda kv: kv[1][0])
        out["dominant"] = dict(kernel=name, us=round(tot / n * 1e3, 2),
                               **fractions(nbytes, flops, tot / n * 1e-3, hbm, bf16))
    return out


def config_block(spec: mi.Spec, world: int) -> dict:
    """The workload description both arms print."""
    return {"workload": spec.name, "B": spec.B, "T": spec.T, "H": spec.H, "d_k": spec.d,
            "d_v": spec.d, "C": spec.C, "inputs": spec.dtype, "state": "fp32",
            "S0_M0": "N(0, %g^2)" % spec.state_std if spec.state_std > 0 else "zero",
            "step": "mdn_chunk_fwd over the batch + 1 mdn_step token",
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": f"replicas x{world} (independent heads, no collective)",
            "global_batch": spec.B * world, "seq_len": spec.T}


def run_ours(args, rank, world, device):
    import momentum_delta_rule_mdn_b200 as mdn

    spec0 = workload_spec(args.workload)
    spec = rank_spec(spec0, rank)
    hbm, bf16, peak_src = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    main = Pass(mdn, spec, device)
    B, T, H, d = spec.B, spec.T, spec.H, spec.d
    clk = ClockSampler(device.index)   # sampled during the timed steps only
    step_ms, kernels = main.time(args.steps, args.warmup, flush, world, clock=clk)
    clocks = clk.summary()
    ms = float(np.mean(step_ms))
    ms_max = max_over_ranks(ms, world, device)
    value = whole_job_value(B * T, world, ms_max)

    # ---- dominant kernel and its roofline: the pass's algorithmic bytes and
    # flops (pass_work) over that kernel's average device time
    nbytes, flops = pass_work(spec)
    roofline = None
    gpu_launches = sum(n for _, n in kernels.values())
    chunk = {k: v for k, v in kernels.items() if k != "step"}
    if chunk:
        name, (tot_ms, n) = max(chunk.items(), key=lambda kv: kv[1][0])
        bound, work, unit = kernel_work(name, spec)
        avg_s = tot_ms / n * 1e-3
        if bound == "hbm":
            achieved, peak = work / avg_s / 1e9, hbm
        else:
            achieved, peak = work / avg_s / 1e12, FP32_ALU_PEAK_TFLOPS
        tr = load_traffic().get(name, {}).get(spec0.name, {})
        traffic = tr.get("bytes_per_launch")
        fr = fractions(nbytes, flops, avg_s, hbm, bf16)
        roofline = {"kernel": name, "bound": bound, "achieved": round(achieved, 3),
                    "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
                    "traffic": traffic,
                    "peak_source": (f"{peak_src} (MEASURED_PEAKS.json: copy GB/s, bf16 burst TFLOP/s)"
                                    if bound != "alu" else
                                    "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz"),
                    "work": {"bytes": int(nbytes), "flops": flops,
                             "per_token_head": {"bytes": (5 * d * (2 if spec.dtype == "bf16" else 4)
                                                          + 16),
                                                "flops": 12 * spec.C * d + 12 * d * d},
                             "states_bytes": int(nbytes - B * T * H * (5 * d * (2 if spec.dtype == "bf16" else 4) + 16))},
                    "tensor": {"achieved_tflops": fr["achieved_tflops"], "peak": bf16,
                               "frac": fr["tensor_frac"]},
                    "roofline_frac": fr["roofline_frac"],
                    "kernel_ms_avg": round(tot_ms / n, 5),
                    "share_of_step": round(tot_ms / args.steps / ms, 4),
                    "step": fractions(nbytes + token_bytes(spec), flops, ms_max * 1e-3, hbm, bf16)}

    # ---- the other workloads, timed the same way (rank 0's batch shapes)
    configs = {}
    if not args.no_side_configs:
        for w in SIDE_WORKLOADS:
            if mi.WORKLOADS[w].name == spec0.name:
                continue
            sp = rank_spec(mi.WORKLOADS[w], rank)
            p = Pass(mdn, sp, device)
            sms, sk = p.time(max(5, min(args.steps, 20)), args.warmup, flush, world)
            configs[sp.name] = pass_summary(sp, float(np.mean(sms)), sk, len(sms), hbm, bf16)
            del p
    main_summary = pass_summary(spec, ms, kernels, args.steps, hbm, bf16)

    # ---- end to end through the public call, host (pinned) buffers
    e2e = None if args.no_e2e else run_e2e(args, mdn, main.inp, main.tok, spec, device, world)
    side = set() if args.no_decode else set(args.side.split(","))
    decode = run_decode(args, mdn, device, hbm) if "decode" in side else None
    gates = run_gate_params(args, mdn, device, hbm, B * T * H) if "gates" in side else None
    varlen = run_varlen(args, mdn, device, spec0) if "varlen" in side else None
    backward = run_backward(args, mdn, device, mi.WORKLOADS[1]) if "backward" in side else None

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if "inter_tc" in kernels else "f32",
        "data": "synthetic (seeded generator; gates from the stable parameterisation)",
        "config": config_block(spec0, world),
        "roofline": roofline,
        "kernels": {k: {"ms_total": round(v[0], 4), "launches": v[1]} for k, v in kernels.items()},
        "gpu_launches": gpu_launches,
        "e2e": e2e,
        "clocks": clocks,
        "headline": main_summary,
        "configs": configs,
    }
    if decode:
        line["decode"] = decode
    if gates:
        line["gate_params"] = gates
    if varlen:
        line["varlen"] = varlen
    if backward:
        line["backward"] = backward
    return line, spec


def run_decode(args, mdn, device, hbm_peak):
    """mdn_step at the decode workload's shape (B=256, H=16, d=128): S and M
    (2 x 268 MB fp32) are read and written once per token, so no L2 flush is
    needed.  Reports tokens/s and the kernel's HBM fraction."""
    spec = mi.WORKLOADS[4]
    B, H, d = spec.B, spec.H, spec.d
    tok = mi.make_inputs(mi.replace(spec, T=1, seed=spec.seed + 11))
    t = {k: v[:, 0].contiguous() for k, v in mi.to_torch(tok, device).items() if v is not None}
    S = torch.randn((B, H, d, d), device=device) * 0.01
    M = torch.randn((B, H, d, d), device=device) * 0.01
    o = torch.empty_like(t["q"])
    gates = ("alpha_log", "mu_log", "beta", "eta")
    for _ in range(3):
        mdn.step(t["q"], t["k"], t["v"], *(t[g] for g in gates), spec.q_corr, S, M, o=o,
                 want_vtilde=False)
    n = max(5, min(args.steps, 50))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(n):
        mdn.step(t["q"], t["k"], t["v"], *(t[g] for g in gates), spec.q_corr, S, M, o=o,
                 want_vtilde=False)
    b.record()
    torch.cuda.synchronize()
    sec = a.elapsed_time(b) / n * 1e-3
    _, bytes_per_step, _ = kernel_work("step", spec)
    gbs = bytes_per_step / sec / 1e9
    # the same token with ||S_t - S_{t-1}||_F per head (memset + step + sqrt)
    ds = torch.empty((B, H), device=device)
    for _ in range(3):
        mdn.step_with_delta_norm(t["q"], t["k"], t["v"], *(t[g] for g in gates), spec.q_corr,
                                 S, M, o=o, ds_norm=ds, want_vtilde=False)
    torch.cuda.synchronize()
    a.record()
    for _ in range(n):
        mdn.step_with_delta_norm(t["q"], t["k"], t["v"], *(t[g] for g in gates), spec.q_corr,
                                 S, M, o=o, ds_norm=ds, want_vtilde=False)
    b.record()
    torch.cuda.synchronize()
    sec_dn = a.elapsed_time(b) / n * 1e-3
    gbs_dn = bytes_per_step / sec_dn / 1e9
    return {"workload": spec.name, "tokens_per_s": round(B / sec, 1),
            "us_per_step": round(sec * 1e6, 2), "achieved_gbs": round(gbs, 1),
            "peak_gbs": hbm_peak, "frac": round(gbs / hbm_peak, 4), "steps": n,
            "with_delta_norm": {"us_per_step": round(sec_dn * 1e6, 2),
                                "achieved_gbs": round(gbs_dn, 1),
                                "frac": round(gbs_dn / hbm_peak, 4)}}


VARLEN_LENGTHS = (3000, 1500, 64, 2500, 1, 700, 300, 127)


def run_varlen(args, mdn, device, spec0):
    """mdn_chunk_fwd_varlen on the workload's token budget (B*T tokens, same H
    and d) split into sequences of mixed lengths (the fixed list above, the
    remainder as a last sequence).  L2 flushed before every timed call, as in
    the main step."""
    total = spec0.B * spec0.T
    lens = []
    for x in VARLEN_LENGTHS:
        if sum(lens) + x <= total:
            lens.append(x)
    if sum(lens) < total:
        lens.append(total - sum(lens))
    H, d = spec0.H, spec0.d
    inp = mi.make_inputs(mi.replace(spec0, B=1, T=total, seed=spec0.seed + 21))
    dev = {k: v[0] for k, v in mi.to_torch(inp, device).items() if v is not None}
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=device)
    N = len(lens)
    lib = mdn.library()
    code = 1 if dev["q"].dtype == torch.bfloat16 else 0
    ws = torch.empty(int(lib.mdn_chunk_fwd_varlen_workspace_size(N, total, H, d, d, spec0.C, code)),
                     dtype=torch.uint8, device=device)
    out = (torch.empty_like(dev["q"]), torch.empty_like(dev["q"]),
           torch.empty((N, H, d, d), device=device), torch.empty((N, H, d, d), device=device))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    gates = ("alpha_log", "mu_log", "beta", "eta")

    def call():
        mdn.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), cu,
                             inp.d_corr, None, None, spec0.C, out=out, workspace=ws)
    for _ in range(3):
        flush.zero_()
        call()
    n = max(5, min(args.steps, 50))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        flush.zero_()
        ev[i][0].record()
        call()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    return {"lengths": lens, "tokens": total, "H": H, "d": d, "ms": round(ms, 5),
            "tokens_per_s": round(total / (ms * 1e-3), 1), "calls": n,
            "includes": "checked offsets, chunk-aligned gather, intra + inter kernels"}


def run_backward(args, mdn, device, spec0):
    """mdn_chunk_bwd at the workload's shape from the forward pass's saved
    vtilde and a random cotangent of o; per-kernel device times from the
    library's events (a separate pass)."""
    inp = mi.make_inputs(spec0)
    dev = mi.to_torch(inp, device)
    gates = ("alpha_log", "mu_log", "beta", "eta")
    B, T, H, d = spec0.B, spec0.T, spec0.H, spec0.d
    o, vt, _, _ = mdn.chunk_fwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates),
                                inp.d_corr)
    do = torch.randn_like(o)
    code = 1 if o.dtype == torch.bfloat16 else 0
    ws = torch.empty(int(mdn.library().mdn_chunk_bwd_workspace_size(B, T, H, d, d, spec0.C, code)),
                     dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call():
        mdn.chunk_bwd(dev["q"], dev["k"], dev["v"], *(dev[g] for g in gates), inp.d_corr, vt,
                      do, workspace=ws)
    for _ in range(2):
        call()
    n = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        flush.zero_()
        ev[i][0].record()
        call()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    mdn.profile_enable(True)
    mdn.profile_read(reset=True)
    for _ in range(n):
        call()
    torch.cuda.synchronize()
    kern = mdn.profile_read(reset=True)
    mdn.profile_enable(False)
    nbytes, flops = bwd_work(spec0)
    hbm, bf16, src = load_peaks()
    roof = {"bound": "latency (serial per-chunk phases; see the kernel times)",
            "work": {"bytes": nbytes, "flops": flops,
                     "per_token_head": {"bytes": int(nbytes // (B * T * H)), "flops": 28 * spec0.C * d + 28 * d * d}},
            **fractions(nbytes, flops, ms * 1e-3, hbm, bf16),
            "peak": {"hbm_gbs": hbm, "bf16_tflops": bf16, "source": src}}
    return {"workload": spec0.name, "ms": round(ms, 4), "tokens_per_s": round(B * T / (ms * 1e-3), 1),
            "calls": n, "roofline": roof,
            "path": ("tcgen05 (bf16, d = 128), fp32 accumulation" if o.dtype == torch.bfloat16 and d == 128
                     else "fp32 CUDA cores"),
            "kernels_ms": {k: round(v[0] / v[1], 4) for k, v in kern.items()}}


def run_gate_params(args, mdn, device, hbm_peak, workload_n: int):
    """K-0 (gates from pre-activations): 16 bytes read + 16 written per
    element.  Timed at the workload's token-head count and at 2^26 elements
    (512 MiB per launch, far above L2) for the HBM fraction.  The launches are
    captured in a CUDA graph and replayed, so host overhead is not timed."""
    out = {}
    reps = 20
    for label, n in (("workload", workload_n), ("hbm", 1 << 26)):
        g = torch.Generator(device=device).manual_seed(5)
        pre = [torch.randn(n, device=device, generator=g) for _ in range(4)]
        res = tuple(torch.empty(n, device=device) for _ in range(4))
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                mdn.gate_params(*pre, s=1.0, mu_log_min=-1.0, out=res)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(reps):
                mdn.gate_params(*pre, s=1.0, mu_log_min=-1.0, out=res)
        graph.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        sec = a.elapsed_time(b) / reps * 1e-3
        gbs = 32.0 * n / sec / 1e9
        out[label] = {"elements": n, "us_per_launch": round(sec * 1e6, 2),
                      "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4)}
        del graph, pre, res
    out["peak_gbs"] = hbm_peak
    out["timing"] = f"CUDA graph of {reps} back-to-back launches, replayed once after a warm replay"
    return out

def run_e2e(args, mdn, inp, tok, spec, device, world):
    """Same metric through the public API with pinned host buffers: every step
    copies its inputs host->device, runs the pass and the decode token, and
    reads every result back (o, vtilde, S_T, M_T after the token, the token's
    o).  Steps are pipelined over three streams with two buffer sets, as a
    serving loop would run them: step i's inputs go in while step i-1
    computes and step i-2's results come out (PCIe carries both directions at
    once).  The timed region spans the first copy in to the last copy out."""
    host = mi.to_torch(inp, "cpu", pin=True)
    htok = {k: (v[:, 0].contiguous().pin_memory() if v is not None else None)
            for k, v in mi.to_torch(tok, "cpu").items()}
    gates = ("alpha_log", "mu_log", "beta", "eta")
    B, T, H, d = spec.B, spec.T, spec.H, spec.d
    keys = [k for k, v in host.items() if v is not None]
    tkeys = [k for k, v in htok.items() if v is not None]
    n = max(3, min(args.steps, 20))
    nb = 2
    din = [{k: torch.empty_like(host[k], device=device) for k in keys} for _ in range(nb)]
    dtk = [{k: torch.empty_like(htok[k], device=device) for k in tkeys} for _ in range(nb)]
    dout = [(torch.empty_like(din[0]["q"]), torch.empty_like(din[0]["q"]),
             torch.empty((B, H, d, d), device=device), torch.empty((B, H, d, d), device=device),
             torch.empty_like(dtk[0]["q"])) for _ in range(nb)]
    hout = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dout[0])
            for _ in range(nb)]
    ws = [torch.empty(mdn.chunk_fwd_workspace_size(B, T, H, d, spec.C, host["q"].dtype),
                      dtype=torch.uint8, device=device) for _ in range(nb)]
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys) + \
        sum(htok[k].numel() * htok[k].element_size() for k in tkeys)
    d2h = sum(t.numel() * t.element_size() for t in hout[0])
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done = [ev() for _ in range(n)]
    cmp_done = [ev() for _ in range(n)]
    out_done = [ev() for _ in range(n)]

    def run(n_steps):
        for i in range(n_steps + 2):
            if i < n_steps:                       # copy in step i
                j = i % nb
                with torch.cuda.stream(s_in):
                    if i >= nb:
                        s_in.wait_event(cmp_done[i - nb])   # its buffers were read
                    for k in keys:
                        din[j][k].copy_(host[k], non_blocking=True)
                    for k in tkeys:
                        dtk[j][k].copy_(htok[k], non_blocking=True)
                    in_done[i].record(s_in)
            if 1 <= i <= n_steps:                 # compute step i - 1
                c = i - 1
                j = c % nb
                s_cmp.wait_event(in_done[c])
                if c >= nb:
                    s_cmp.wait_event(out_done[c - nb])      # its results were read out
                o, vt, S_T, M_T, o1 = dout[j]
                x, t = din[j], dtk[j]
                mdn.chunk_fwd(x["q"], x["k"], x["v"], *(x[g] for g in gates), inp.d_corr,
                              x.get("S0"), x.get("M0"), spec.C, out=(o, vt, S_T, M_T),
                              workspace=ws[j], stream=s_cmp)
                mdn.step(t["q"], t["k"], t["v"], *(t[g] for g in gates), inp.d_corr, S_T, M_T,
                         o=o1, want_vtilde=False, stream=s_cmp)
                cmp_done[c].record(s_cmp)
            if i >= 2:                            # copy out step i - 2
                c = i - 2
                j = c % nb
                with torch.cuda.stream(s_out):
                    s_out.wait_event(cmp_done[c])
                    for dst, src in zip(hout[j], dout[j]):
                        dst.copy_(src, non_blocking=True)
                    out_done[c].record(s_out)

    run(min(n, max(1, args.warmup)))
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    s_cmp.wait_stream(s_in)
    s_out.wait_stream(s_in)
    run(n)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / n, world, device)
    return {"value": round(B * T * world / (ms * 1e-3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n,
            "pipeline": "copy-in, compute, copy-out streams; two buffer sets"}


# ---------------------------------------------------------------- CPU oracle
def cpu_baseline(spec: mi.Spec, inp=None, budget_s: float = 10.0):
    """The fp64 oracle as it stands, on the host cores, over the same workload
    (the whole batch per repetition), repeated until ~budget_s of CPU work."""
    import oracle
    inp = inp or mi.make_inputs(spec)
    args = (inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta, inp.eta, inp.d_corr,
            inp.S0, inp.M0)
    args64 = [None if a is None else (np.asarray(a, dtype=np.float64) if isinstance(a, np.ndarray) else a)
              for a in args]
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.chunk_fwd(*args64)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(spec.B * spec.T / dt, 1), "unit": "tokens/s",
            "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{spec.name}: the full batch ({spec.B}x{spec.T} tokens x {spec.H} heads, "
                      f"fp64 stepwise recurrence), {reps} repetition(s), {dt:.2f} s each",
            "seconds_per_batch": round(dt, 3)}


def run_reference(args, rank, world):
    """The reference arm: the oracle timed on the host cores, rank 0 only."""
    if rank != 0:
        return None
    import oracle
    spec = workload_spec(args.workload)
    inp = mi.make_inputs(spec)
    tok = decode_token(spec, spec.seed + 1)
    c64 = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    full = [c64(x) for x in (inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta, inp.eta)]
    s0, m0 = c64(inp.S0), c64(inp.M0)
    # bounded sample per step: the first `hs` heads of every batch row
    t0 = time.perf_counter()
    oracle.chunk_fwd(*[x[:, :, :1] for x in full], inp.d_corr,
                     None if s0 is None else s0[:, :1], None if m0 is None else m0[:, :1])
    per_head = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)   # whole run within ~2.5 minutes
    hs = int(max(1, min(spec.H, budget / max(per_head, 1e-6))))

    def one():
        o, vt, S, M = oracle.chunk_fwd(*[x[:, :, :hs] for x in full], inp.d_corr,
                                       None if s0 is None else s0[:, :hs],
                                       None if m0 is None else m0[:, :hs])
        oracle.step(*[c64(x)[:, 0, :hs] for x in (tok.q, tok.k, tok.v, tok.alpha_log,
                                                  tok.mu_log, tok.beta, tok.eta)],
                    inp.d_corr, S, M)

    for _ in range(args.warmup):
        one()
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        one()
        times.append(time.perf_counter() - t)
    sec = float(np.mean(times))
    tokens = spec.B * spec.T * hs / spec.H          # token-heads processed / heads per token
    value = tokens / sec
    cb = {"value": round(value, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
          "kind": "oracle",
          "sample": f"{spec.name}: {hs} of {spec.H} heads per batch row each step "
                    f"(token rate scaled by {hs}/{spec.H})"}
    return {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(spec, world),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- plumbing
def workload_spec(w):
    if w is None:
        return mi.WORKLOADS[DEFAULT_WORKLOAD]
    if str(w).isdigit():
        return mi.WORKLOADS[int(w)]
    for s in mi.WORKLOADS:
        if s.name == w:
            return s
    raise SystemExit(f"unknown workload {w!r}")


def rank_spec(spec0: mi.Spec, rank: int) -> mi.Spec:
    """The workload of one rank: same shape, its own seed (ranks are replicas
    over independent batches; no two ranks draw the same inputs)."""
    return mi.replace(spec0, seed=spec0.seed + 7919 * rank)


def whole_job_value(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Weak-scaling throughput: the tokens every rank processed over the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="config name or index (default: 2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip every side measurement")
    ap.add_argument("--side", default="decode,gates,varlen,backward",
                    help="side measurements after the timed step (comma list of decode, gates, "
                         "varlen, backward)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-side-configs", action="store_true",
                    help="skip timing the other workloads beside the headline one")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        line, spec = run_ours(args, rank, world, device)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(spec)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
