"""Benchmark of the Jano hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload large]
                    [--impl reference] [--no-cpu-baseline] [--no-e2e] [--no-next]

One step = one pass of the whole hot path over one batch of synthetic input
(block scores over the latent history, level split of the per-token field,
the 50-step schedule, KV-cache scatter of the Active tokens' fresh K/V and
active-query attention over the whole cache), all through the C ABI.

Metric: active-query attention TFLOP/s, FLOPs = 4 * N_act * N * d * heads,
divided by the whole step's device time (max over ranks); the analyzer and
scatter HBM GB/s and per-kernel times are reported beside it.  Every rank
runs an independent replica of the workload (a different seed): the path
has no data-path exchange, so N GPUs process N problems ("weak" scaling).

Beside the step (not in its value) the line reports ``next_rows``: the
block's projections on the step's active tokens -- the fused Q/K/V projection
writing K/V straight into the cache and the output projection scattered back
to the token rows -- with their TFLOP/s, the FFT baseline score with the
analyzer timed under the same conditions (HBM GB/s), and the attention at
the schedule's larger due sets (Active + Moderate, and every token).

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on
a bounded sample of the same workload, extrapolated stage by stage to the
full workload.

Other measurements, each printing its own JSON line (``--mode``):

    --workload schedule50     the 50-step interleaved schedule with the KV cache
                              carried across steps, against 50 full steps, and the
                              active-fraction sweep on the same shape
    --mode splits             attention TFLOP/s for every key-split count of a few
                              due sets (the data the split choice was fitted to)
    --mode sharded            per-rank work of the head-sharded step, one rank at a
                              time on this GPU (W = --ranks)
    --mode projection         the projections of the active rows alone
    --mode spectral           the FFT baseline score beside the analyzer and a
                              plain read, L2 cleaned before each launch
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "active-query attn TFLOP/s (% BF16 peak) at 75.6K tokens; analyzer HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def n_active_of(w) -> int:
    """Due tokens of the step the bench times (the first interleaved step:
    the Active level, frac_active of the tokens in basis points, floored)."""
    return int(round(w.frac_active * 10000)) * w.n_tokens // 10000


def workload_config(w, world: int = 1):
    """The `config` of the JSON line: the same dict for both arms."""
    cache_gb = 2.0 * w.n_tokens * w.heads * w.d * 2 / 1e9
    act_gb = 3.0 * n_active_of(w) * w.heads * w.d * 2 / 1e9
    return {
        "workload": f"{w.name}: latent {list(w.latent_shape)} fp32, blocks {list(w.block)}, "
                    f"{w.n_tokens} tokens x {w.heads} heads x d={w.d} BF16, "
                    f"levels {round(w.frac_active*100)}/{round((1-w.frac_active-w.frac_static)*100)}/"
                    f"{round(w.frac_static*100)} from a smooth token field, Active-only step",
        "tokens": w.n_tokens, "heads": w.heads, "d": w.d,
        "latent": list(w.latent_shape), "block": list(w.block), "patch": list(w.patch),
        "schedule": {"T": w.T, "warmup": w.warmup, "cooldown": w.cooldown,
                     "period_moderate": w.period_moderate, "period_static": w.period_static},
        "n_active": n_active_of(w), "global_batch": world, "parallelism": f"replicas x{world}",
        "l2": f"no flush: the per-step working set (K/V cache {cache_gb:.2f} GB, Q/K/V act "
              f"{act_gb:.2f} GB) is larger than the 126 MB L2",
    }


def host_cores() -> int:
    """Host threads this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


# ------------------------------------------------------------------ ranks
def max_over_ranks(x: float, dist=None, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a group);
    a CUDA tensor for NCCL, a CPU tensor otherwise."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Aggregate throughput: every rank processes its own replica."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ inputs
def make_inputs(w, seed_shift=0):
    import synth
    import torch
    TF, TH, TW = w.grid
    lat = synth.latent_history(w.K, w.C, w.F, w.H, w.W, seed=w.seed + seed_shift)
    field = synth.token_field(TF, TH, TW, seed=(w.seed + seed_shift) * 10 + 1, sigma=w.field_sigma)
    N = w.n_tokens
    n_cap = int(round(w.frac_active * 10000)) * N // 10000
    base = (w.seed + seed_shift) * 1000
    inp = dict(lat=torch.from_numpy(lat), field=torch.from_numpy(field),
               q_act=synth.normal_bf16((n_cap, w.heads, w.d), base + 1),
               k_act=synth.normal_bf16((n_cap, w.heads, w.d), base + 2),
               v_act=synth.normal_bf16((n_cap, w.heads, w.d), base + 3))
    k_cache = synth.normal_bf16((N, w.heads, w.d), base + 4)
    v_cache = synth.normal_bf16((N, w.heads, w.d), base + 5)
    return inp, k_cache, v_cache, n_cap


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        busy = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


# ------------------------------------------------------------------ traffic record
def traffic_for(kernel_src_rel, workload):
    """DRAM bytes per launch from the committed ncu record, if it was taken on
    the current source of that kernel and on this workload; else None."""
    rec = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, kernel_src_rel)
    if not (os.path.exists(rec) and os.path.exists(src)):
        return None
    with open(rec) as fh:
        d = json.load(fh)
    ent = d.get(kernel_src_rel)
    if not ent:
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if ent.get("source_sha") != sha or ent.get("workload_key") != workload:
        return None
    return ent.get("bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle
def oracle_inputs(inp, k_cache, v_cache, n_act):
    """BF16 bit arrays of the step's inputs for the CPU oracle (made once)."""
    import synth
    return {"kb": synth.bits_of(k_cache), "vb": synth.bits_of(v_cache),
            "qb": synth.bits_of(inp["q_act"][:n_act]), "ka": synth.bits_of(inp["k_act"]),
            "va": synth.bits_of(inp["v_act"])}


def _oracle_attention_rows(bits, rows, threads):
    """oracle.active_attention on `rows`, cut into chunks run by `threads`
    host threads (each chunk is the unchanged single-threaded oracle; ctypes
    releases the GIL around the C call)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    if threads <= 1:
        return oracle.active_attention(bits["qb"], bits["kb"], bits["vb"], rows=rows)
    parts = np.array_split(rows, min(threads, rows.size))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        outs = list(ex.map(lambda r: oracle.active_attention(bits["qb"], bits["kb"], bits["vb"], rows=r),
                           parts))
    return np.concatenate(outs, axis=0)


def cpu_oracle_step_time(w, inp, bits, attn_rows, threads=1, rng_seed=0):
    """Time the oracle stage by stage: block scores, classify, schedule and
    the KV scatter over the full workload, attention on `attn_rows` sampled
    active rows (all heads, all keys) spread over `threads` host threads,
    extrapolated linearly to every active row.  Returns a dict with the
    extrapolated seconds per full step, the step's FLOPs, the wall time of
    the sampled step and a text describing the sample.  `bits` holds the BF16
    bit arrays of oracle_inputs (the scatter writes into its caches)."""
    import oracle
    oracle.build()
    N, H, d = w.n_tokens, w.heads, w.d
    lat = inp["lat"].numpy()
    field = inp["field"].numpy()
    t_all = time.perf_counter()
    t = time.perf_counter()
    oracle.block_scores(lat, w.block)
    lv = oracle.classify(field, w.frac_active, w.frac_static)
    off, idx, _ = oracle.build_schedule(lv, (w.F, w.H, w.W), w.patch, w.patch, w.T, w.warmup,
                                        w.cooldown, w.period_moderate, w.period_static)
    n_act = int(off[w.warmup + 1] - off[w.warmup])
    sel = idx[off[w.warmup]:off[w.warmup + 1]]
    oracle.kv_scatter(bits["ka"][:n_act], bits["va"][:n_act], sel, bits["kb"], bits["vb"], inplace=True)
    est = time.perf_counter() - t
    g = np.random.default_rng(rng_seed)
    rows = np.sort(g.choice(n_act, size=min(attn_rows, n_act), replace=False)).astype(np.int32)
    t = time.perf_counter()
    _oracle_attention_rows(bits, rows, threads)
    dt = time.perf_counter() - t
    est += dt * n_act / rows.size
    return {"seconds": est, "flops": 4.0 * n_act * N * d * H, "wall_s": time.perf_counter() - t_all,
            "sample": f"block scores, classify, schedule and scatter over the full workload; "
                      f"attention on {rows.size} of {n_act} active rows x {H} heads x {N} keys, "
                      f"extrapolated to every active row (fp64 C oracle, {threads} host "
                      f"thread{'s' if threads > 1 else ''})"}


def cpu_baseline(w, inp, bits, cores, rng_seed=0):
    """The oracle on all host cores (attention rows over a thread pool) and
    single-threaded, each on a bounded sample (tens of seconds at most)."""
    multi = cpu_oracle_step_time(w, inp, bits, attn_rows=min(512, max(16, 4 * cores)), threads=cores,
                                 rng_seed=rng_seed)
    single = cpu_oracle_step_time(w, inp, bits, attn_rows=4, threads=1, rng_seed=rng_seed + 1)
    return {"value": multi["flops"] / multi["seconds"] / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "sample": multi["sample"], "extrapolated": True,
            "full_step_s_extrapolated": multi["seconds"], "wall_s": multi["wall_s"],
            "single_thread": {"value": single["flops"] / single["seconds"] / 1e12, "unit": "TFLOP/s",
                              "cores": 1, "sample": single["sample"], "extrapolated": True,
                              "full_step_s_extrapolated": single["seconds"], "wall_s": single["wall_s"]}}


def measure_projections(J, hp, step, stream, pk, reps=10, cpu_rows=0):
    """The block's projections on the step's active tokens (outside the hot
    path's step, reported beside it): the fused Q/K/V projection that writes
    K/V straight into the cache, and the output projection scattered back to
    the token rows.  Random-init weights N(0, 1/k) in BF16; hidden states
    N(0, 1) for every token (hidden size heads x d)."""
    import torch
    start, n_act = hp.due(step)
    idx = hp.idx[start:start + n_act]
    N, hd = hp.N, hp.heads * hp.d
    g = torch.Generator(device=hp.dev).manual_seed(1234)
    x = torch.randn((N, hd), generator=g, device=hp.dev).to(torch.bfloat16)
    w_qkv = (torch.randn((3 * hd, hd), generator=g, device=hp.dev) * hd ** -0.5).to(torch.bfloat16)
    w_o = (torch.randn((hd, hd), generator=g, device=hp.dev) * hd ** -0.5).to(torch.bfloat16)
    q = torch.empty((n_act, hd), dtype=torch.bfloat16, device=hp.dev)
    o_act = torch.randn((n_act, hd), generator=g, device=hp.dev).to(torch.bfloat16)
    y = torch.zeros((N, hd), dtype=torch.bfloat16, device=hp.dev)
    kc, vc = hp.k_cache.view(N, hd), hp.v_cache.view(N, hd)
    ops = {
        "qkv_project": (lambda: J.qkv_project(x, idx, w_qkv, q, kc, vc, stream), 2.0 * n_act * 3 * hd * hd),
        "out_proj_scatter": (lambda: J.gather_gemm(o_act, w_o, y, scatter=idx, stream=stream),
                             2.0 * n_act * hd * hd),
    }
    res = {}
    for name, (fn, flops) in ops.items():
        for _ in range(3):
            fn()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        evs[0].record(stream)
        for i in range(reps):
            fn()
            evs[i + 1].record(stream)
        stream.synchronize()
        ms = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(reps))[reps // 2]
        tf = flops / (ms * 1e-3) / 1e12
        res[name] = {"ms": ms, "TFLOP/s": tf, "flops": flops, "frac_of_burst_peak": tf / pk["bf16_tflops"],
                     "shape": {"m": n_act, "n": (3 if name == "qkv_project" else 1) * hd, "k": hd}}
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in projections: {J.jano_status_str(code)}")
    if cpu_rows:
        # the fp64 CPU oracle on a bounded sample: cpu_rows active rows of the
        # fused projection, extrapolated to all n_act rows
        import oracle
        import synth
        oracle.build()
        rows = idx[:cpu_rows].cpu().numpy()
        xb = synth.bits_of(x[torch.from_numpy(rows).long().to(hp.dev)].cpu())
        wb = synth.bits_of(w_qkv.cpu())
        t0 = time.perf_counter()
        oracle.gather_gemm(xb, wb)
        dt = (time.perf_counter() - t0) * n_act / cpu_rows
        fl = res["qkv_project"]["flops"]
        res["qkv_project"]["cpu_oracle"] = {
            "TFLOP/s": fl / dt / 1e12, "cores": 1, "kind": "oracle",
            "sample": f"{cpu_rows} of {n_act} rows x {3 * hd} outputs x k={hd} "
                      "(single-threaded fp64 C, extrapolated)"}
    return res


def measure_attention_sizes(J, hp, stream, pk, reps=3):
    """Attention over the same cache at the step's larger due sets (outside
    the step, reported beside it): an interleaved step where Active and
    Moderate tokens are due, and a full step (every token due, e.g. warm-up),
    with random BF16 queries.  TFLOP/s as for the headline."""
    import torch
    N, H, d = hp.N, hp.heads, hp.d
    o = hp.host_offsets
    step_am = next((t for t in range(hp.sched.warmup, hp.sched.T - hp.sched.cooldown)
                    if o[t + 1] - o[t] > o[hp.sched.warmup + 1] - o[hp.sched.warmup]), None)
    cases = {"full": (0, o[1] - o[0])}
    if step_am is not None:
        cases["active_moderate"] = (o[step_am], o[step_am + 1] - o[step_am])
    g = torch.Generator(device=hp.dev).manual_seed(4321)
    q = torch.randn((N, H, d), generator=g, device=hp.dev).to(torch.bfloat16)
    out = torch.empty((N, H, d), dtype=torch.bfloat16, device=hp.dev)
    res = {}
    for name, (start, n) in cases.items():
        idx = hp.idx[start:start + n]
        qn = q[:n]
        fn = lambda: J.attention_auto(qn, hp.k_cache, hp.v_cache, idx, n, N, H, d, out, stream, hp.att_ws)
        fn()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        evs[0].record(stream)
        for i in range(reps):
            fn()
            evs[i + 1].record(stream)
        stream.synchronize()
        ms = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(reps))[reps // 2]
        flops = 4.0 * n * N * d * H
        tf = flops / (ms * 1e-3) / 1e12
        res[f"attention_{name}"] = {"ms": ms, "TFLOP/s": tf, "n_active": n, "flops": flops,
                                    "frac_of_sustained_peak": tf / pk.get("bf16_tflops_sustained", pk["bf16_tflops"])}
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in the attention sizes: {J.jano_status_str(code)}")
    return res


def measure_fft_score(J, hp, stream, pk, reps=10, cutoff=1):
    """The FFT baseline score (outside the step, reported beside it) against
    the analyzer under the same conditions: each launch alone, L2 cleaned
    before it (a 256 MB read, which leaves no dirty lines to write back), on
    the last warm-up snapshot x_K.  The FFT score reads one snapshot; the
    analyzer reads all K+1.  The one-pass read ceiling of the analyzer's bytes
    (jano_stream_sum, a kernel that only streams them) and a plain torch.sum,
    timed the same way, give the rate a single pass of that size reaches."""
    import torch
    K, C = hp.K, hp.C
    x = hp.lat[K]
    out = torch.empty_like(hp.scores)
    geom = hp.lg.c()
    flush = torch.ones(64 << 20, dtype=torch.float32, device=hp.dev)
    sms = torch.cuda.get_device_properties(hp.dev).multi_processor_count
    partial = torch.empty(sms, dtype=torch.float32, device=hp.dev)
    snap_bytes = float(x.numel()) * 4 + out.numel() * 4
    lat_bytes = float(hp.lat.numel()) * 4 + out.numel() * 4
    ops = {
        "fft_score": (lambda: J.jano_fft_scores(x, C, geom, cutoff, out, stream), snap_bytes),
        "block_scores_same_conditions": (lambda: J.jano_block_scores(hp.lat, K, C, geom, hp.w_t, hp.w_s,
                                                                     out, stream), lat_bytes),
        "plain_read_same_bytes": (lambda: torch.sum(hp.lat), float(hp.lat.numel()) * 4),
        "stream_read_same_bytes": (lambda: J.jano_stream_sum(hp.lat, hp.lat.numel(), partial, sms, stream),
                                   float(hp.lat.numel()) * 4),
    }
    res = {}
    for name, (fn, nbytes) in ops.items():
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        ms = []
        for _ in range(reps):
            with torch.cuda.stream(stream):
                flush.sum()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
            stream.synchronize()
            ms.append(a.elapsed_time(b))
        m = sorted(ms)[reps // 2]
        gbs = nbytes / (m * 1e-3) / 1e9
        res[name] = {"ms": m, "GB/s": gbs, "frac_of_hbm": gbs / pk["hbm_gbs"], "algorithmic_bytes": nbytes}
    res["fft_score"]["cutoff"] = cutoff
    # the analyzer against the one-pass read ceiling of the same bytes (a kernel
    # that only streams them: jano_stream_sum), both timed the same way
    res["block_scores_same_conditions"]["frac_of_stream_read"] = (
        res["stream_read_same_bytes"]["ms"] / res["block_scores_same_conditions"]["ms"])
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in the FFT score: {J.jano_status_str(code)}")
    return res


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    inp, k_cache, v_cache, n_cap = make_inputs(w)
    bits = oracle_inputs(inp, k_cache, v_cache, n_cap)
    cores = host_cores()
    # attention rows per sampled step: sized so that the whole run stays
    # within a few minutes (about 2 s of one core per row of the large step)
    rows = args.ref_rows if args.ref_rows > 0 else \
        max(1, min(512, (90 * cores) // (2 * max(1, args.steps + args.warmup))))
    est, walls = [], []
    res = None
    for i in range(args.warmup + args.steps):
        res = cpu_oracle_step_time(w, inp, bits, attn_rows=rows, threads=cores, rng_seed=i)
        if i >= args.warmup:
            est.append(res["seconds"])
            walls.append(res["wall_s"])
        log(f"reference step {i}: sampled step {res['wall_s']:.1f} s, "
            f"extrapolated full step {res['seconds']:.1f} s")
    t = statistics.mean(est)
    value = res["flops"] / t / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            # what was run and timed: one sampled step (the value comes from
            # its per-stage extrapolation to the full step, given beside it)
            "ms_per_step": statistics.mean(walls) * 1e3, "ms_per_step_kind": "sampled step (wall)",
            "extrapolated": True, "full_step_ms_extrapolated": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, world), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": res["sample"], "extrapolated": True},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, w, rank, world, local_rank, dist):
    import torch
    import kv_cache_analyzer_b200 as J
    from kv_cache_analyzer_b200.pipeline import HostStepper, HotPath, KERNELS_PER_STEP

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(dev)
    pk, pk_src = peaks()

    inp, k_cache, v_cache, n_cap = make_inputs(w, seed_shift=rank)
    hp = HotPath(K=w.K, C=w.C, latent_geom=J.Geometry(w.F, w.H, w.W, w.block, w.patch),
                 token_geom=J.Geometry(w.F, w.H, w.W, w.patch, w.patch), heads=w.heads, d=w.d,
                 frac_active=w.frac_active, frac_static=w.frac_static,
                 sched=J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static),
                 device=dev, stream=stream)
    hp.set_activations(n_cap)
    with torch.cuda.stream(stream):
        hp.lat.copy_(inp["lat"])
        hp.field.copy_(inp["field"])
        hp.q_act.copy_(inp["q_act"]); hp.k_act.copy_(inp["k_act"]); hp.v_act.copy_(inp["v_act"])
        hp.k_cache.copy_(k_cache); hp.v_cache.copy_(v_cache)
    stream.synchronize()
    hp.plan()
    step = w.warmup                       # first interleaved step: Active tokens only
    _, n_act = hp.due(step)
    assert n_act <= n_cap, (n_act, n_cap)
    flops = 4.0 * n_act * w.n_tokens * w.d * w.heads

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- warm-up
    for _ in range(args.warmup):
        hp.run_step_kernels(step)
    stream.synchronize()
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error after warm-up: {J.jano_status_str(code)}")

    # ---- timed: device-resident inputs, per-stage events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        start.record(stream)
        for i in range(args.steps):
            hp.run_step_kernels(step, evs[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    total_ms = start.elapsed_time(end)
    stage = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(5)] for e in evs])  # ms
    # stage columns: scores, classify, schedule, scatter, attention
    stage_ms = stage.mean(axis=0)
    t_max = max_over_ranks(total_ms, dist, dev)
    ms_per_step = t_max / args.steps
    value = whole_job_tflops(flops, world, ms_per_step)
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in timed region: {J.jano_status_str(code)}")

    # ---- end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        host = {k: v.pin_memory() for k, v in inp.items()}
        host["q_act"] = host["q_act"][:n_act]; host["k_act"] = host["k_act"][:n_act]
        host["v_act"] = host["v_act"][:n_act]
        host_out = torch.empty(hp.out.shape, dtype=hp.out.dtype).pin_memory()
        own = {k: getattr(hp, k) for k in HostStepper.IN_KEYS + ("out",)}
        stepper = HostStepper(hp, host, host_out)
        stepper.run(step, max(1, args.warmup))
        torch.cuda.synchronize(dev)
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        stepper.run(step, args.steps, start=s2, end=e2)
        torch.cuda.synchronize(dev)
        barrier()
        hp.use(own)
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), dist, dev)
        e2e = {"value": whole_job_tflops(flops, world, e2e_ms / args.steps), "unit": "TFLOP/s",
               "h2d_bytes_per_step": HotPath.h2d_bytes(host),
               "d2h_bytes_per_step": host_out.numel() * host_out.element_size()}

    # ---- the same step replayed from a CUDA graph, and the launch-bound plan
    # kernels timed in graphs of back-to-back launches (every rank alike)
    graph = None
    if not args.no_graph:
        graph = measure_graphs(J, hp, step, stream, args.steps, flops, world, dist, dev)

    if rank != 0:
        return 0

    # ---- per-kernel figures and roofline of the dominant kernel (attention)
    hbm = pk["hbm_gbs"]
    bf16_sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    lat_bytes = float(np.prod(w.latent_shape)) * 4
    scat_bytes = 4.0 * n_act * w.heads * w.d * 2
    att_tflops = flops / (stage_ms[4] * 1e-3) / 1e12
    kernels = {
        "block_scores": {"ms": stage_ms[0], "GB/s": lat_bytes / (stage_ms[0] * 1e-3) / 1e9,
                         "algorithmic_bytes": lat_bytes},
        "classify": {"ms": stage_ms[1], "n": w.n_tokens},
        "build_schedule": {"ms": stage_ms[2], "T": w.T},
        "kv_scatter": {"ms": stage_ms[3], "GB/s": scat_bytes / (stage_ms[3] * 1e-3) / 1e9,
                       "algorithmic_bytes": scat_bytes},
        "active_attention": {"ms": stage_ms[4], "TFLOP/s": att_tflops, "flops": flops,
                             "n_active": n_act},
    }
    for k in ("block_scores", "kv_scatter"):
        kernels[k]["frac_of_hbm"] = kernels[k]["GB/s"] / hbm
    if graph is not None:
        kernels["classify"]["graph_us"] = graph.pop("classify_us")
        kernels["build_schedule"]["graph_us"] = graph.pop("build_schedule_us")
    kernels["active_attention"]["frac_of_burst_peak"] = att_tflops / pk["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": att_tflops, "peak": bf16_sus, "unit": "TFLOP/s",
                "frac": att_tflops / bf16_sus,
                "traffic": traffic_for("kv_cache_analyzer_b200/csrc/attention.cu", w.name),
                "peak_kind": f"{pk_src} sustained cuBLAS bf16 (kernel timed inside a long step)",
                "kernel": "active_attention"}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        bits = oracle_inputs(inp, k_cache, v_cache, n_cap)
        cpu = cpu_baseline(w, inp, bits, host_cores())

    next_rows = None
    if not args.no_next:
        next_rows = measure_projections(J, hp, step, stream, pk,
                                        cpu_rows=0 if args.no_cpu_baseline or world > 1 else 2)
        next_rows.update(measure_fft_score(J, hp, stream, pk))
        # the analyzer's one-pass ceiling beside its in-step figure
        kernels["block_scores"]["stream_read_ceiling_GB/s"] = next_rows["stream_read_same_bytes"]["GB/s"]
        kernels["block_scores"]["frac_of_stream_read_alone"] = \
            next_rows["block_scores_same_conditions"]["frac_of_stream_read"]
        next_rows.update(measure_attention_sizes(J, hp, stream, pk))

    cfg = workload_config(w, world)
    assert cfg["n_active"] == n_act, (cfg["n_active"], n_act)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": (KERNELS_PER_STEP + (1 if hp.last_split > 1 else 0)) * args.steps, "clocks": clk.summary(),
            "kernels": kernels, "graph": graph, "next_rows": next_rows,
            "peaks": {"source": pk_src, "hbm_gbs": hbm,
                                          "bf16_tflops": pk["bf16_tflops"],
                                          "bf16_tflops_sustained": bf16_sus}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ other measurements
def measure_graphs(J, hp, step, stream, steps, flops, world, dist, dev, repeat=20, reps=5):
    """The step captured once as a CUDA graph and replayed `steps` times (no
    host launches; device time by events on the stream, max over ranks), and
    classify and the schedule each captured as `repeat` back-to-back
    launches (per launch: replay time / repeat; their inputs are a few
    hundred KB, resident in L2 after the first launch, as in the step)."""
    import torch
    g = hp.capture_step(step)
    cls = hp.capture_repeated(
        lambda s: J.jano_classify(hp.field, hp.field.numel(), hp.frac_active, hp.frac_static, hp.levels, s),
        repeat)
    sch = hp.capture_repeated(
        lambda s: J.jano_build_schedule(hp.levels, hp._tgc, hp._sc, hp.offsets, hp.idx, hp.idx.numel(),
                                        hp.token_levels, hp.ws, hp.ws_bytes, s),
        repeat)

    def replay_ms(graph, n):
        with torch.cuda.stream(stream):
            for _ in range(3):
                graph.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                graph.replay()
            b.record(stream)
        stream.synchronize()
        return a.elapsed_time(b)

    step_ms = max_over_ranks(replay_ms(g, steps), dist, dev) / steps
    cls_us = replay_ms(cls, reps) / (reps * repeat) * 1e3
    sch_us = replay_ms(sch, reps) / (reps * repeat) * 1e3
    _raise_device_error(J, stream, "graph replays")
    del g, cls, sch
    return {"step_ms": step_ms, "TFLOP/s": whole_job_tflops(flops, world, step_ms), "replays": steps,
            "classify_us": cls_us, "build_schedule_us": sch_us, "launches_per_graph": repeat,
            "note": "the timed step replayed from one CUDA graph; classify and schedule per launch "
                    "inside graphs of back-to-back launches (no host work between launches)"}



def _events_ms(fn, stream, reps, warm=2, pick="median"):
    """Device time of fn() on `stream` by CUDA events (after `warm` calls)."""
    import torch
    for _ in range(warm):
        fn()
    ms = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        stream.synchronize()
        ms.append(a.elapsed_time(b))
    return min(ms) if pick == "min" else sorted(ms)[len(ms) // 2]


def _raise_device_error(J, stream, what):
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in {what}: {J.jano_status_str(code)}")


def run_schedule50(args):
    """The 50-step interleaved schedule of the 32,760-token x 12-head workload
    (5 warm-up, Moderate every 2, Static every 4, 5 cool-down), each step the
    KV scatter of its due tokens into the carried cache and their attention
    over the whole cache, against 50 full steps; then the active-fraction
    sweep (attention of the top fraction of the token field).  Fresh
    activations of a step come from seeded device pools by the indexing rule
    of synth.step_rows."""
    import torch
    import synth
    import kv_cache_analyzer_b200 as J
    w = synth.WORKLOADS["schedule50"]
    N, H, d = w.n_tokens, w.heads, w.d
    dev = torch.device("cuda")
    st = torch.cuda.current_stream()
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    sched = J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static)
    lat = torch.from_numpy(synth.latent_history(w.K, w.C, w.F, w.H, w.W, seed=w.seed)).to(dev)
    levels = J.classify(J.block_scores(lat, geom), w.frac_active, w.frac_static)
    off, idx, _ = J.build_schedule(levels, geom, sched)
    off_h = off.cpu().tolist()                       # one read-back per generation
    g = torch.Generator(device=dev).manual_seed(5000)
    pool = [torch.randn(N, H, d, device=dev, generator=g).bfloat16() for _ in range(3)]
    kc = torch.randn(N, H, d, device=dev, generator=g).bfloat16()
    vc = torch.randn(N, H, d, device=dev, generator=g).bfloat16()
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device=dev)
    ws = J.SplitWorkspace(dev)

    def attend(q, toks, n):
        J.attention_auto(q, kc, vc, toks, n, N, H, d, out, st, ws)

    def run(tok_lists):
        evs = []
        for s, toks in enumerate(tok_lists):
            rows = (toks.long() + 7 * s) % N
            q, k, v = pool[0][rows], pool[1][rows], pool[2][rows]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            J.kv_scatter(k, v, toks, kc, vc)
            attend(q, toks, toks.numel())
            b.record(st)
            evs.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    sched_lists = [idx[off_h[s]:off_h[s + 1]] for s in range(w.T)]
    all_toks = torch.arange(N, dtype=torch.int32, device=dev)
    run(sched_lists)
    sched_ms = min(run(sched_lists) for _ in range(args.reps))
    run([all_toks] * w.T)
    full_ms = min(run([all_toks] * w.T) for _ in range(args.reps))
    due = np.diff(np.array(off_h))
    sched_flops = 4.0 * float(due.sum()) * N * d * H
    full_flops = 4.0 * w.T * N * N * d * H

    TF, TH, TW = w.grid
    fld = torch.from_numpy(synth.token_field(TF, TH, TW, seed=w.seed * 10 + 1, sigma=w.field_sigma)).to(dev)
    tgeom = J.Geometry(w.F, w.H, w.W, w.patch, w.patch)
    sweep = []
    for f in [float(x) for x in args.fractions.split(",")]:
        lv = J.classify(fld, f, 1.0 - f)
        # periods longer than the schedule: the first interleaved step holds only Active tokens
        o, ix, _ = J.build_schedule(lv, tgeom, J.Schedule(w.T, w.warmup, w.cooldown, 10 * w.T, 10 * w.T))
        a0, a1 = o[w.warmup:w.warmup + 2].cpu().tolist()
        toks, n_act = ix[a0:a1], a1 - a0
        q = pool[0][:n_act]
        ms = _events_ms(lambda: attend(q, toks, n_act), st, args.reps, pick="min")
        sweep.append({"fraction": f, "n_active": n_act, "ms": ms,
                      "key_split": J.jano_active_attention_splits(n_act, N, H, d),
                      "TFLOP/s": 4.0 * n_act * N * d * H / (ms * 1e-3) / 1e12})
    _raise_device_error(J, st, "the schedule50 run")
    print(json.dumps({
        "mode": "schedule50",
        "workload": f"schedule50: {N} tokens x {H} heads x d={d} BF16, 30/30/40 levels, T=50",
        "schedule_ms": sched_ms, "full_ms": full_ms, "speedup_vs_full": full_ms / sched_ms,
        "flop_ratio_full_over_schedule": full_flops / sched_flops,
        "schedule_tflops": sched_flops / (sched_ms * 1e-3) / 1e12,
        "full_tflops": full_flops / (full_ms * 1e-3) / 1e12,
        "due_token_steps": int(due.sum()), "sweep": sweep}), flush=True)
    return 0


SPLIT_CASES = [(32760, 12, n) for n in (1638, 3276, 8190, 16380, 24570, 32760)] + \
              [(75600, 5, 18900), (75600, 40, 18900), (75600, 40, 41580)]


def run_splits(args):
    """Attention TFLOP/s for every key-split count of a few due sets (keys,
    heads, due queries; d = 128; random BF16 cache and queries, due rows a
    random sorted subset), with the library's own choice beside them."""
    import torch
    import kv_cache_analyzer_b200 as J
    d = 128
    dev = torch.device("cuda")
    st = torch.cuda.current_stream()
    cases = [tuple(c) for c in args.case] if args.case else SPLIT_CASES
    for N, H, n in cases:
        g = torch.Generator(device=dev).manual_seed(0)
        kc = torch.randn((N, H, d), generator=g, device=dev).bfloat16()
        vc = torch.randn((N, H, d), generator=g, device=dev).bfloat16()
        q = torch.randn((n, H, d), generator=g, device=dev).bfloat16()
        idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:n]).values.int()
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=dev)
        line = {"mode": "splits", "keys": N, "heads": H, "n_act": n,
                "chosen": J.jano_active_attention_splits(n, N, H, d), "TFLOP/s": {}}
        for z in args.splits:
            if z > (N + 127) // 128:
                continue
            ws = torch.empty(max(16, J.jano_active_attention_workspace_bytes(n, H, d, z)),
                             dtype=torch.uint8, device=dev)
            ms = _events_ms(lambda: J.active_attention(q, kc, vc, idx, out, split=z, workspace=ws),
                            st, args.reps)
            line["TFLOP/s"][z] = round(4.0 * n * N * d * H / (ms * 1e-3) / 1e12, 1)
        _raise_device_error(J, st, "the split sweep")
        print(json.dumps(line), flush=True)
        del kc, vc, q, out
    return 0


def run_sharded(args):
    """Per-rank work of the head-sharded step (frame slabs for the analyzer,
    head ranges for scatter and attention), measured one rank at a time on
    this GPU: each rank's block scores, then (after the ranks' scores are
    joined by a copy standing in for the all-gather, not timed) classify,
    schedule, scatter and attention.  Random device inputs of the large
    workload's shapes (--frames/--height/--width/--heads shrink it).  One
    JSON line per W: every rank's time, the slowest, and T_1 / (W T_W)."""
    import torch
    import kv_cache_analyzer_b200 as J
    from kv_cache_analyzer_b200.sharding import ShardedHotPath
    K, C, F, H, W = 5, 16, args.frames, args.height, args.width
    heads, d = args.heads, 128
    frac_active, frac_static = 0.25, 0.45
    lg = J.Geometry(F, H, W, (1, 4, 4), (1, 2, 2))
    tg = J.Geometry(F, H, W, (1, 2, 2), (1, 2, 2))
    sched = J.Schedule(50, 5, 5, 2, 4)
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
        for sh in shards:
            sh.run_local_scores()
        with torch.cuda.stream(stream):
            full = torch.cat([sh.local_scores() for sh in shards])
            for sh in shards:
                sh.scores.copy_(full)
        for sh in shards:
            sh.run_after_gather()
        stream.synchronize()
        for sh in shards:
            sh.host_offsets = sh.offsets.cpu().tolist()
        n_act = shards[0].due(step)[1]
        per_rank = []
        for sh in shards:
            t_scores = _events_ms(sh.run_local_scores, stream, args.reps)

            def rest(sh=sh):
                sh.run_after_gather()
                sh.run_head_kernels(step)
            t_rest = _events_ms(rest, stream, args.reps)
            per_rank.append({"rank": sh.rank, "heads": sh.heads, "frames": sh.f_own,
                             "key_split": sh.last_split, "ms": t_scores + t_rest, "scores_ms": t_scores})
        _raise_device_error(J, stream, "the sharded ranks")
        t_max = max(p["ms"] for p in per_rank)
        if base is None and world == 1:
            base = t_max
        line = {"mode": "sharded", "ranks": world, "n_active": n_act, "max_rank_ms": t_max,
                "per_rank": per_rank}
        if base is not None:
            line["t1_over_w_tw"] = base / (world * t_max)
        print(json.dumps(line), flush=True)
        del shards
        torch.cuda.empty_cache()
    return 0


def run_projection(args):
    """The projections of the active rows alone: random BF16 hidden states
    x [N][D] (N(0, 1)), weights W_qkv [3D][D] and W_o [D][D] (N(0, 1/D)), M
    distinct active tokens; the fused Q/K/V projection (K and V straight into
    the token-ordered cache) and the output projection scattered back."""
    import torch
    import kv_cache_analyzer_b200 as J
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
    ops = {"qkv_project": (lambda: J.qkv_project(x, idx, w_qkv, q, kc, vc), 2.0 * M * 3 * D * D),
           "out_proj_scatter": (lambda: J.gather_gemm(o_act, w_o, y, scatter=idx), 2.0 * M * D * D)}
    res = {"mode": "projection", "shape": {"tokens": N, "hidden": D, "active": M}}
    for name, (fn, flops) in ops.items():
        ms = _events_ms(fn, st, args.reps, warm=3)
        res[name] = {"ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12}
    _raise_device_error(J, st, "the projections")
    print(json.dumps(res), flush=True)
    return 0


def run_spectral(args):
    """The FFT baseline score of the last snapshot, the analyzer's block
    scores over all K+1 snapshots and a plain torch.sum over the analyzer's
    bytes, each launch alone with the L2 cleaned (a 256 MB read) before it,
    on a random fp32 latent history (default: the large video latent)."""
    import torch
    import kv_cache_analyzer_b200 as J
    C, F, H, W, K = args.channels, args.frames, args.height, args.width, 5
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    lat = torch.randn((K + 1, C, F, H, W), generator=g, device=dev)
    geom = J.Geometry(F, H, W, (1, 4, 4), (1, 1, 1))
    out = torch.empty(geom.n_blocks, device=dev)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()
    gc = geom.c()
    snap = lat[K]
    ops = {"fft_score": (lambda: J.jano_fft_scores(snap, C, gc, 1, out, st),
                         4.0 * (snap.numel() + out.numel())),
           "block_scores": (lambda: J.jano_block_scores(lat, K, C, gc, 0.5, 0.5, out, st),
                            4.0 * (lat.numel() + out.numel())),
           "plain_read": (lambda: torch.sum(lat), 4.0 * lat.numel())}
    res = {"mode": "spectral", "shape": {"channels": C, "frames": F, "height": H, "width": W,
                                          "block": [1, 4, 4], "steps": K, "cutoff": 1,
                                          "n_blocks": geom.n_blocks}}
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
    _raise_device_error(J, st, "the spectral run")
    print(json.dumps(res), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="large")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="attention rows per oracle sample of --impl reference (0: sized from "
                         "--steps/--warmup so the run ends within minutes)")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replays of the step")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the projections measured beside the step")
    ap.add_argument("--mode", default="step",
                    choices=["step", "schedule50", "splits", "sharded", "projection", "spectral"],
                    help="step: the hot path's step (the contract line); others: see the docstring "
                         "(--workload schedule50 selects schedule50)")
    ap.add_argument("--reps", type=int, default=5, help="repetitions of the other modes")
    ap.add_argument("--fractions", default="0.1,0.25,0.5,0.75,1.0", help="schedule50: sweep points")
    ap.add_argument("--splits", type=int, nargs="+", default=[1, 2, 3, 4, 5, 6, 7, 8, 10, 12])
    ap.add_argument("--case", type=int, nargs=3, action="append", metavar=("N", "HEADS", "N_ACT"),
                    help="splits: a due set (repeatable)")
    ap.add_argument("--ranks", type=int, nargs="+", default=[1, 2, 4, 8], help="sharded: W values")
    ap.add_argument("--frames", type=int, default=21)
    ap.add_argument("--height", type=int, default=90)
    ap.add_argument("--width", type=int, default=160)
    ap.add_argument("--heads", type=int, default=40)
    ap.add_argument("--channels", type=int, default=16, help="spectral: latent channels")
    ap.add_argument("--tokens", type=int, default=75600, help="projection: tokens")
    ap.add_argument("--hidden", type=int, default=5120, help="projection: hidden size")
    ap.add_argument("--active", type=int, default=18900, help="projection: active rows")
    args = ap.parse_args()

    if args.workload == "schedule50" and args.mode == "step":
        args.mode = "schedule50"
    if args.mode != "step":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "mode": args.mode,
                              "unavailable": "the reference arm times the hot path's step only"}))
            return 0
        return {"schedule50": run_schedule50, "splits": run_splits, "sharded": run_sharded,
                "projection": run_projection, "spectral": run_spectral}[args.mode](args)

    import synth
    w = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        return run_gpu(args, w, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
