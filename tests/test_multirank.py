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


# ---------------------------------------------------------------- head / frame sharding
def test_partitions_cover_everything_once():
    from kv_cache_analyzer_b200.sharding import frame_block_range, head_range, slab_frames
    for world in (1, 2, 3, 8):
        for heads in (1, 12, 40):
            got = [h for r in range(world) for h in range(*head_range(r, world, heads))]
            assert got == list(range(heads))
        for F, bf in ((21, 1), (21, 2), (4, 1), (1, 1)):
            n_fb = -(-F // bf)
            got = [b for r in range(world) for b in range(*frame_block_range(r, world, n_fb))]
            assert got == list(range(n_fb))
            frames = []
            for r in range(world):
                f0, own, slab = slab_frames(r, world, F, bf)
                frames += list(range(f0, f0 + own))
                assert slab == (own + (1 if f0 + own < F else 0) if own else 0)
            assert frames == list(range(F))


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import numpy as np
        import oracle
        import synth
        from kv_cache_analyzer_b200.sharding import frame_block_range, slab_frames, torch_all_gather
        K, C, F, H, W, block = 4, 3, 5, 8, 12, (1, 4, 4)
        lat = synth.latent_history(K, C, F, H, W, seed=9)
        f0, own, slab = slab_frames(rank, world, F, block[0])
        n_fb = F
        per_fb = (H // 4) * (W // 4)
        counts = [(frame_block_range(r, world, n_fb)[1] - frame_block_range(r, world, n_fb)[0]) * per_fb
                  for r in range(world)]
        # this rank's blocks, scored on its slab with the halo frame (the oracle
        # stands in for the kernel on the CPU ranks)
        if slab:
            local = torch.from_numpy(oracle.block_scores(np.ascontiguousarray(lat[:, :, f0:f0 + slab]), block))
        else:
            local = torch.zeros(0, dtype=torch.float64)         # a rank without frame-blocks
        full = torch.empty(sum(counts), dtype=torch.float64)
        torch_all_gather(local[:counts[rank]].contiguous(), full, counts)
        out[rank] = full.numpy().tobytes()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 7])
def test_sharded_scores_gather_to_the_whole_latent(world):
    # frame slabs with one halo frame, scored per rank and all-gathered, give
    # the scores of the whole latent exactly (uneven slabs with 3 ranks)
    import numpy as np
    import oracle
    import synth
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    ref = oracle.block_scores(synth.latent_history(4, 3, 5, 8, 12, seed=9), (1, 4, 4))
    for r in range(world):
        got = np.frombuffer(out[r], dtype=np.float64)
        np.testing.assert_array_equal(got, ref)
