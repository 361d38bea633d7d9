"""The N-GPU host logic of bench.py, run as two gloo ranks on the CPU:
every rank times its own replica, the whole-job number divides all ranks'
work by the slowest rank's time, and only rank 0 runs the reference arm."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_ms = [30.0, 45.0][rank]                  # rank 1 is slower
        t = bench.max_over_ranks(local_ms, dist)
        v = bench.whole_job_tflops(29.26e12, world, t / 10)
        # the reference arm: rank 0 alone works; the others return at once
        class A:
            warmup, steps, ref_rows = 0, 1, 1
        rc = bench.run_reference(A, None, rank, world) if rank != 0 else 0
        out[rank] = (t, v, rc)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_by_the_slowest():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        t, v, rc = out[r]
        assert t == 45.0                               # max over ranks on every rank
        assert v == pytest.approx(2 * 29.26e12 / 4.5e-3 / 1e12)
        assert rc == 0


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(12.5, None) == 12.5
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)   # 1e12 FLOP in 1 ms
