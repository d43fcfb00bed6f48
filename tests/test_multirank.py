"""The multi-rank path of bench.py on CPU: two gloo ranks, as torch.distributed.run
would start them on two GPUs.  Each rank is a replica over its own seeded batch
(heads are independent, so there is no collective on the data path); the only
collectives are the barrier and the max over ranks of the step time."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import argparse

    import bench
    import mdn_inputs as mi
    import oracle

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        spec = bench.rank_spec(mi.WORKLOADS[0], rank)
        inp = mi.make_inputs(spec)
        # each replica runs the pass on its own batch (the oracle stands in for the GPU path)
        o, vt, S, M = oracle.chunk_fwd(inp.q, inp.k, inp.v, inp.alpha_log, inp.mu_log, inp.beta,
                                       inp.eta, inp.d_corr, inp.S0, inp.M0)
        checksum = torch.tensor([float(np.abs(o).sum())], dtype=torch.float64)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, checksum)
        bench.barrier(world)
        step_ms = 1.0 + rank  # rank 1 is the slowest
        ms_max = bench.max_over_ranks(step_ms, world, torch.device("cpu"))
        value = bench.whole_job_value(spec.B * spec.T, world, ms_max)
        ref = bench.run_reference(argparse.Namespace(workload=0, steps=1, warmup=0), rank, world)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([ms_max, value, sums[0].item(), sums[1].item(), spec.seed,
                          0.0 if ref is None else 1.0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    # the step time is the max over ranks, seen identically by both
    assert r0[0] == r1[0] == 2.0
    # whole-job throughput: both ranks' tokens over the slowest rank's time
    assert r0[1] == pytest.approx(1 * 256 * 2 / 2.0e-3)
    # the two replicas drew different batches (different seeds, different outputs)
    assert r0[4] != r1[4]
    assert r0[2] == r1[2] and r0[3] == r1[3] and r0[2] != r0[3]
    # the reference arm runs on rank 0 only; the other ranks exit without work
    assert r0[5] == 1.0 and r1[5] == 0.0
