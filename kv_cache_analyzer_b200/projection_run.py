"""Timing of the projections of the active rows.

    python -m kv_cache_analyzer_b200.projection_run [--tokens N] [--hidden D] [--active M] [--reps R]

Random BF16 hidden states x [N][D] (N(0, 1)), weights W_qkv [3D][D] and
W_o [D][D] (N(0, 1/D)), M distinct active tokens.  Times, with CUDA events on
the current stream after three warm-up calls, the fused Q/K/V projection
(jano_qkv_project: Q to the active rows, K and V straight into the
token-ordered cache) and the output projection scattered back to the token
rows (jano_gather_gemm), and prints one JSON line with their TFLOP/s.
Defaults: the large video step (75,600 tokens, hidden 5,120, 18,900 active).
"""
from __future__ import annotations

import argparse
import json

import torch

from . import device_error, gather_gemm, jano_status_str, qkv_project


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=75600)
    ap.add_argument("--hidden", type=int, default=5120)
    ap.add_argument("--active", type=int, default=18900)
    ap.add_argument("--reps", type=int, default=10)
    args = ap.parse_args(argv)
    N, D, M = args.tokens, args.hidden, args.active
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    x = torch.randn((N, D), generator=g, device=dev).to(torch.bfloat16)
    w_qkv = (torch.randn((3 * D, D), generator=g, device=dev) * D ** -0.5).to(torch.bfloat16)
    w_o = (torch.randn((D, D), generator=g, device=dev) * D ** -0.5).to(torch.bfloat16)
    idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:M]).values.to(torch.int32)
    q = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((N, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    o_act = torch.randn((M, D), generator=g, device=dev).to(torch.bfloat16)
    y = torch.zeros((N, D), dtype=torch.bfloat16, device=dev)
    st = torch.cuda.current_stream()
    ops = {"qkv_project": (lambda: qkv_project(x, idx, w_qkv, q, kc, vc), 2.0 * M * 3 * D * D),
           "out_proj_scatter": (lambda: gather_gemm(o_act, w_o, y, scatter=idx), 2.0 * M * D * D)}
    res = {"shape": {"tokens": N, "hidden": D, "active": M}}
    for name, (fn, flops) in ops.items():
        for _ in range(3):
            fn()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.reps + 1)]
        evs[0].record(st)
        for i in range(args.reps):
            fn()
            evs[i + 1].record(st)
        torch.cuda.synchronize()
        ms = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.reps))[args.reps // 2]
        res[name] = {"ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12}
    code = device_error()
    if code:
        raise RuntimeError(jano_status_str(code))
    print(json.dumps(res))


if __name__ == "__main__":
    main()
