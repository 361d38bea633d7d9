"""Per-rank work of the head-sharded step, measured one rank at a time.

    python -m kv_cache_analyzer_b200.sharding_run [--ranks 1 2 4 8] [--reps R]
        [--frames F] [--height H] [--width W] [--heads N]

Builds the step of the large video workload by default (latent
[6][16][21][90][160] fp32 with 1x4x4 blocks, 75,600 tokens x 40 heads x
d=128 BF16, 25/30/45 level split, first interleaved step = the 18,900
Active tokens; the size flags shrink it) from random
device inputs, cuts it into W ranks with ``ShardedHotPath`` (frame slabs for
the analyzer, head ranges for scatter and attention) and times each rank's
kernels alone on this GPU with CUDA events: its block scores, then (after the
scores of all ranks are joined by a copy, which stands in for the
all-gather and is not timed) classify, schedule, scatter and attention.
Prints one JSON line per W with every rank's time, the slowest rank's, and
the ratio T_1 / (W T_W) that strong scaling over W GPUs would reach if the
all-gather of the block scores (4 bytes per block) were free.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import Geometry, Schedule, device_error, jano_status_str
from .sharding import ShardedHotPath


def _time(fn, stream, reps):
    for _ in range(2):
        fn()
    ms = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        stream.synchronize()
        ms.append(a.elapsed_time(b))
    return sorted(ms)[reps // 2]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--ranks", type=int, nargs="+", default=[1, 2, 4, 8])
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--frames", type=int, default=21)
    ap.add_argument("--height", type=int, default=90)
    ap.add_argument("--width", type=int, default=160)
    ap.add_argument("--heads", type=int, default=40)
    args = ap.parse_args(argv)
    K, C, F, H, W = 5, 16, args.frames, args.height, args.width
    heads, d = args.heads, 128
    frac_active, frac_static = 0.25, 0.45
    lg = Geometry(F, H, W, (1, 4, 4), (1, 2, 2))
    tg = Geometry(F, H, W, (1, 2, 2), (1, 2, 2))
    sched = Schedule(50, 5, 5, 2, 4)
    step = sched.warmup
    N = tg.n_tokens
    n_cap = int(round(frac_active * 10000)) * N // 10000
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    lat = torch.randn((K + 1, C, F, H, W), generator=g, device=dev)
    field = torch.rand(tg.n_blocks, generator=g, device=dev)
    acts = {k: torch.randn((n_cap, heads, d), generator=g, device=dev).to(torch.bfloat16)
            for k in ("q_act", "k_act", "v_act")}
    kc = torch.randn((N, heads, d), generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn((N, heads, d), generator=g, device=dev).to(torch.bfloat16)
    stream = torch.cuda.Stream()
    base = None
    for world in args.ranks:
        shards = []
        for r in range(world):
            sh = ShardedHotPath(rank=r, world=world, K=K, C=C, latent_geom=lg, token_geom=tg,
                                heads=heads, d=d, frac_active=frac_active, frac_static=frac_static,
                                sched=sched, stream=stream, all_gather=None)
            sh.set_activations(n_cap)
            sh.load_latent(lat)
            with torch.cuda.stream(stream):
                sh.field.copy_(field)
                for k, v in acts.items():
                    getattr(sh, k).copy_(sh.head_slice(v))
                sh.k_cache.copy_(sh.head_slice(kc))
                sh.v_cache.copy_(sh.head_slice(vc))
            shards.append(sh)

        def join():
            full = torch.cat([sh.local_scores() for sh in shards])
            for sh in shards:
                sh.scores.copy_(full)

        # the plan once, to learn the due lists
        for sh in shards:
            sh.run_local_scores()
        with torch.cuda.stream(stream):
            join()
        for sh in shards:
            sh.run_after_gather()
        stream.synchronize()
        for sh in shards:
            sh.host_offsets = sh.offsets.cpu().tolist()
        n_act = shards[0].due(step)[1]

        per_rank = []
        for sh in shards:
            t_scores = _time(sh.run_local_scores, stream, args.reps)

            def rest(sh=sh):
                sh.run_after_gather()
                sh.run_head_kernels(step)
            t_rest = _time(rest, stream, args.reps)
            per_rank.append({"rank": sh.rank, "heads": sh.heads, "frames": sh.f_own,
                             "ms": t_scores + t_rest, "scores_ms": t_scores})
        code = device_error()
        if code:
            raise RuntimeError(jano_status_str(code))
        t_max = max(p["ms"] for p in per_rank)
        if base is None and world == 1:
            base = t_max
        line = {"ranks": world, "n_active": n_act, "max_rank_ms": t_max, "per_rank": per_rank}
        if base is not None:
            line["t1_over_w_tw"] = base / (world * t_max)
        print(json.dumps(line), flush=True)
        del shards
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
