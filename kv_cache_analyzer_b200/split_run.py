"""Attention throughput for every key split of a few due-set shapes.

    python -m kv_cache_analyzer_b200.split_run [--reps R] [--splits Z ...]
        [--case N HEADS N_ACT ...]

For each case (keys N, heads, due queries N_ACT; d = 128, BF16 N(0, 1)
random cache and queries, due rows a random sorted subset) times the
attention with every split count Z (`active_attention(..., split=Z)`,
CUDA events on the current stream, median of R after two warm-up calls) and
prints one JSON line: the library's own choice (`jano_active_attention_splits`)
and the TFLOP/s (4 N_ACT N d heads per launch) of each Z.
Default cases: the active-fraction sweep of the 32,760-token x 12-head
workload (5 to 100% due), a 5-head rank of the 75,600-token step split over
8 GPUs, and the 75,600-token x 40-head step's Active and Active + Moderate
due sets.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import active_attention, device_error, jano_active_attention_splits, \
    jano_active_attention_workspace_bytes, jano_status_str

DEFAULT_CASES = [(32760, 12, n) for n in (1638, 3276, 8190, 16380, 24570, 32760)] + \
                [(75600, 5, 18900), (75600, 40, 18900), (75600, 40, 41580)]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--splits", type=int, nargs="+", default=[1, 2, 3, 4, 5, 6, 7, 8, 10, 12])
    ap.add_argument("--case", type=int, nargs=3, action="append", metavar=("N", "HEADS", "N_ACT"))
    args = ap.parse_args(argv)
    cases = args.case or DEFAULT_CASES
    d = 128
    dev = torch.device("cuda")
    st = torch.cuda.current_stream()
    for N, H, n in cases:
        g = torch.Generator(device=dev).manual_seed(0)
        kc = torch.randn((N, H, d), generator=g, device=dev).bfloat16()
        vc = torch.randn((N, H, d), generator=g, device=dev).bfloat16()
        q = torch.randn((n, H, d), generator=g, device=dev).bfloat16()
        idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:n]).values.int()
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=dev)
        line = {"keys": N, "heads": H, "n_act": n, "chosen": jano_active_attention_splits(n, N, H, d),
                "TFLOP/s": {}}
        for z in args.splits:
            if z > (N + 127) // 128:
                continue
            ws = torch.empty(max(16, jano_active_attention_workspace_bytes(n, H, d, z)), dtype=torch.uint8,
                             device=dev)
            fn = lambda: active_attention(q, kc, vc, idx, out, split=z, workspace=ws)
            for _ in range(2):
                fn()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.reps + 1)]
            evs[0].record(st)
            for i in range(args.reps):
                fn()
                evs[i + 1].record(st)
            torch.cuda.synchronize()
            ms = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.reps))[args.reps // 2]
            line["TFLOP/s"][z] = round(4.0 * n * N * d * H / (ms * 1e-3) / 1e12, 1)
        code = device_error()
        if code:
            raise RuntimeError(jano_status_str(code))
        print(json.dumps(line), flush=True)
        del kc, vc, q, out


if __name__ == "__main__":
    main()
