"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

The hot path shards over (batch, head) with no exchange, so a multi-GPU run is one seeded
replica per rank; the job's time is the slowest rank's and its throughput counts every
rank's work.  These tests run that logic in a real two-process gloo group.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from long_context_exact_fwd_b200.workloads import WORKLOADS
    ws, r, local = bench._dist_env()
    w = bench.rank_workload(WORKLOADS["s16k_fwd_bwd"], rank)
    my_ms = [125.0, 250.0][rank]            # rank 1 is the slow one
    mx = bench.max_over_ranks(my_ms)
    value = bench.job_tflops(1e12, 10, mx, ws)
    # the reference arm: only rank 0 works, the others return 0 at once
    class A:
        sample_rows = 0
        warmup = 0
        steps = 0
        gpus = world
    rc = bench.run_reference(A(), WORKLOADS["s16k_fwd_bwd"]) if rank == 1 else 0
    out[rank] = (ws, r, local, w.seed, mx, value, rc)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gloo_group_max_time_and_job_throughput():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    (ws0, r0, l0, seed0, mx0, v0, rc0), (ws1, r1, l1, seed1, mx1, v1, rc1) = res[0], res[1]
    assert (ws0, r0, l0) == (2, 0, 0) and (ws1, r1, l1) == (2, 1, 1)
    assert seed0 != seed1                       # distinct replicas, no shared data
    assert mx0 == mx1 == 250.0                  # every rank sees the slowest rank's time
    # 2 ranks x 10 steps x 1e12 FLOP in 250 ms = 80 TFLOP/s, on every rank
    assert abs(v0 - 80.0) < 1e-9 and abs(v1 - 80.0) < 1e-9
    assert rc1 == 0


def test_single_process_helpers_without_a_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_tflops(2e12, 5, 1000.0, 1) == pytest.approx(10.0)
