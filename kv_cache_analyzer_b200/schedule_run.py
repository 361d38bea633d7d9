"""Timing of a whole interleaved schedule and of an active-fraction sweep.

    python -m kv_cache_analyzer_b200.schedule_run [--fractions 0.1,0.25,0.5,0.75,1.0]

Workload: 32,760 tokens (latent 16 x 21 x 60 x 104, 1x2x2 patches), 12 heads,
d = 128, BF16.  The analyzer scores token-sized blocks of the latent history,
classify splits them 30/30/40, and the schedule covers T = 50 steps (5
warm-up, Moderate every 2, Static every 4, 5 cool-down).  Each step scatters
the fresh K/V of its due tokens into the carried cache and runs attention of
their queries over the whole cache (split over key ranges where the
library's choice for that due set says so).  Reported, as one JSON line:

* the 50 steps' scatter + attention device time, against 50 full-attention
  steps (every token due) on the same shape, and the FLOP ratio;
* attention TFLOP/s at each active fraction of the sweep (top fraction of a
  smooth per-token field).

Fresh activations for a step come from seeded device pools by the indexing
rule of ``synth.step_rows`` (gathered before each step's timed kernels).
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np
import torch

from . import (Geometry, Schedule, active_attention, block_scores, build_schedule, classify,
               device_error, jano_status_str, kv_scatter)


def _timed(fn, stream):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    fn()
    b.record(stream)
    return a, b


def main(argv=None):
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if here not in sys.path:
        sys.path.insert(0, here)
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--fractions", default="0.1,0.25,0.5,0.75,1.0")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    w = synth.WORKLOADS["schedule50"]
    N, H, d = w.n_tokens, w.heads, w.d
    dev = torch.device("cuda")
    st = torch.cuda.current_stream()
    geom = Geometry(w.F, w.H, w.W, w.block, w.patch)
    sched = Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static)

    lat = torch.from_numpy(synth.latent_history(w.K, w.C, w.F, w.H, w.W, seed=w.seed)).to(dev)
    levels = classify(block_scores(lat, geom), w.frac_active, w.frac_static)
    off, idx, _ = build_schedule(levels, geom, sched)
    off_h = off.cpu().tolist()                       # one read-back per generation
    g = torch.Generator(device=dev).manual_seed(5000)
    pool = [torch.randn(N, H, d, device=dev, generator=g).bfloat16() for _ in range(3)]
    kc = torch.randn(N, H, d, device=dev, generator=g).bfloat16()
    vc = torch.randn(N, H, d, device=dev, generator=g).bfloat16()
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device=dev)

    def step_inputs(s):
        toks = idx[off_h[s]:off_h[s + 1]]
        rows = (toks.long() + 7 * s) % N
        return toks, pool[0][rows], pool[1][rows], pool[2][rows]

    # ---- 50 interleaved steps (scatter + attention), cache carried
    def run_schedule():
        evs = []
        for s in range(w.T):
            toks, q, k, v = step_inputs(s)
            evs.append(_timed(lambda: (kv_scatter(k, v, toks, kc, vc), active_attention(q, kc, vc, toks, out)), st))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    run_schedule()                                   # warm-up
    sched_ms = min(run_schedule() for _ in range(args.reps))
    # ---- 50 full steps on the same shape: every token due
    all_toks = torch.arange(N, dtype=torch.int32, device=dev)

    def run_full():
        evs = []
        for s in range(w.T):
            rows = (all_toks.long() + 7 * s) % N
            q, k, v = pool[0][rows], pool[1][rows], pool[2][rows]
            evs.append(_timed(lambda: (kv_scatter(k, v, all_toks, kc, vc), active_attention(q, kc, vc, all_toks, out)), st))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    run_full()
    full_ms = min(run_full() for _ in range(args.reps))
    due = np.diff(np.array(off_h))
    sched_flops = 4.0 * float(due.sum()) * N * d * H
    full_flops = 4.0 * w.T * N * N * d * H

    # ---- active-fraction sweep (attention only)
    TF, TH, TW = w.grid
    fld = torch.from_numpy(synth.token_field(TF, TH, TW, seed=w.seed * 10 + 1, sigma=w.field_sigma)).to(dev)
    tgeom = Geometry(w.F, w.H, w.W, w.patch, w.patch)
    sweep = []
    for f in [float(x) for x in args.fractions.split(",")]:
        lv = classify(fld, f, 1.0 - f)
        # periods longer than the schedule: the first interleaved step holds only Active tokens
        o, ix, _ = build_schedule(lv, tgeom, Schedule(w.T, w.warmup, w.cooldown, 10 * w.T, 10 * w.T))
        a0, a1 = o[w.warmup:w.warmup + 2].cpu().tolist()
        toks = ix[a0:a1]
        n_act = a1 - a0
        q = pool[0][:n_act]
        for _ in range(2):
            active_attention(q, kc, vc, toks, out)
        ts = []
        for _ in range(args.reps):
            a, b = _timed(lambda: active_attention(q, kc, vc, toks, out), st)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = min(ts)
        sweep.append({"fraction": f, "n_active": n_act, "ms": ms,
                      "TFLOP/s": 4.0 * n_act * N * d * H / (ms * 1e-3) / 1e12})
    code = device_error()
    if code:
        raise RuntimeError(jano_status_str(code))
    print(json.dumps({
        "workload": f"schedule50: {N} tokens x {H} heads x d={d} BF16, 30/30/40 levels, T=50",
        "schedule_ms": sched_ms, "full_ms": full_ms, "speedup_vs_full": full_ms / sched_ms,
        "flop_ratio_full_over_schedule": full_flops / sched_flops,
        "schedule_tflops": sched_flops / (sched_ms * 1e-3) / 1e12,
        "full_tflops": full_flops / (full_ms * 1e-3) / 1e12,
        "due_token_steps": int(due.sum()), "sweep": sweep}))


if __name__ == "__main__":
    main()
