"""Timing of the FFT baseline score against the analyzer.

    python -m kv_cache_analyzer_b200.spectral_run [--channels C] [--frames F] [--height H]
        [--width W] [--block BF BH BW] [--steps K] [--cutoff U] [--reps R]

A random fp32 latent history [K+1][C][F][H][W] (N(0, 1)) on the device.
Times, with CUDA events on the current stream after three warm-up calls and
with the L2 cleaned (a 256 MB read) before every launch, the FFT score of
the last snapshot (jano_fft_scores: one snapshot read), the analyzer's block
scores (jano_block_scores: all K+1 snapshots read) and, for scale, a plain
torch.sum over the analyzer's bytes, and prints one JSON line with each
launch's time and HBM GB/s over its algorithmic bytes.
Defaults: the large video latent (C=16, 21 x 90 x 160, 1x4x4 blocks, K=5).
"""
from __future__ import annotations

import argparse
import json

import torch

from . import (Geometry, device_error, jano_block_scores, jano_fft_scores, jano_status_str)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--channels", type=int, default=16)
    ap.add_argument("--frames", type=int, default=21)
    ap.add_argument("--height", type=int, default=90)
    ap.add_argument("--width", type=int, default=160)
    ap.add_argument("--block", type=int, nargs=3, default=(1, 4, 4))
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--cutoff", type=int, default=1)
    ap.add_argument("--reps", type=int, default=10)
    args = ap.parse_args(argv)
    C, F, H, W, K = args.channels, args.frames, args.height, args.width, args.steps
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    lat = torch.randn((K + 1, C, F, H, W), generator=g, device=dev)
    geom = Geometry(F, H, W, tuple(args.block), (1, 1, 1))
    out = torch.empty(geom.n_blocks, device=dev)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()
    gc = geom.c()
    snap = lat[K]
    ops = {"fft_score": (lambda: jano_fft_scores(snap, C, gc, args.cutoff, out, st),
                         4.0 * (snap.numel() + out.numel())),
           "block_scores": (lambda: jano_block_scores(lat, K, C, gc, 0.5, 0.5, out, st),
                            4.0 * (lat.numel() + out.numel())),
           "plain_read": (lambda: torch.sum(lat), 4.0 * lat.numel())}
    res = {"shape": {"channels": C, "frames": F, "height": H, "width": W, "block": list(args.block),
                     "steps": K, "cutoff": args.cutoff, "n_blocks": geom.n_blocks}}
    for name, (fn, nbytes) in ops.items():
        for _ in range(3):
            fn()
        ms = []
        for _ in range(args.reps):
            flush.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        m = sorted(ms)[args.reps // 2]
        res[name] = {"ms": m, "GB/s": nbytes / (m * 1e-3) / 1e9, "algorithmic_bytes": nbytes}
    code = device_error()
    if code:
        raise RuntimeError(jano_status_str(code))
    print(json.dumps(res))


if __name__ == "__main__":
    main()
