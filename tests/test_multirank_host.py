"""The N > 1 host logic of bench.py, run as two gloo ranks on the CPU.

The GEMM does not shard: bench.py runs one independent replica per GPU with
no collective on the data path, times each rank on its own stream and takes
the maximum over ranks. These tests exercise that reduction and the
whole-job aggregation without a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, _ = bench.dist_env()
        assert (r, w) == (rank, world)
        # each replica ran 10 steps of 2 TFLOP; rank 1 was slower
        elapsed = 1.0 + rank
        job = bench.replica_throughput(2e12, 10, elapsed, world)
        mx = bench.max_over_ranks(0.5 * (rank + 3), world)
        bench.barrier(world)
        results[rank] = (job["elapsed_s"], job["tflops"], job["ms_per_step"], mx)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:   # no fork of this multi-threaded process
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        out = dict(results)
    for rank in range(world):
        elapsed, tflops, ms, mx = out[rank]
        assert elapsed == 2.0                      # the slowest rank's time
        assert tflops == pytest.approx(world * 2e12 * 10 / 2.0 / 1e12)
        assert ms == pytest.approx(200.0)
        assert mx == 2.0                           # max of 1.5 and 2.0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    job = bench.replica_throughput(1e12, 4, 2.0, 1)
    assert job["tflops"] == pytest.approx(2.0)
    assert bench.max_over_ranks(3.0, 1) == 3.0


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm prints from rank 0; other ranks exit without work."""
    sys.path.insert(0, ROOT)
    import types

    import bench
    args = types.SimpleNamespace(steps=3, warmup=3)
    assert bench.run_reference(args, rank=1, world=2) is None
