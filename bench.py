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


def workload_config(w):
    return {
        "workload": f"{w.name}: latent {list(w.latent_shape)} fp32, blocks {list(w.block)}, "
                    f"{w.n_tokens} tokens x {w.heads} heads x d={w.d} BF16, "
                    f"levels {round(w.frac_active*100)}/{round((1-w.frac_active-w.frac_static)*100)}/"
                    f"{round(w.frac_static*100)} from a smooth token field, Active-only step",
        "tokens": w.n_tokens, "heads": w.heads, "d": w.d,
        "latent": list(w.latent_shape), "block": list(w.block), "patch": list(w.patch),
        "schedule": {"T": w.T, "warmup": w.warmup, "cooldown": w.cooldown,
                     "period_moderate": w.period_moderate, "period_static": w.period_static},
    }


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


def cpu_oracle_step_time(w, inp, bits, budget_rows=8, rng_seed=0):
    """Time the oracle stage by stage on a bounded sample, extrapolate each
    stage to the full workload; returns (seconds per full step, FLOPs, sample
    text).  `bits` holds the BF16 bit arrays of oracle_inputs (the scatter
    writes into its caches in place)."""
    import oracle
    oracle.build()
    N, H, d = w.n_tokens, w.heads, w.d
    lat = inp["lat"].numpy()
    field = inp["field"].numpy()
    est = 0.0
    parts = []
    # a1 on one frame-block slab of all snapshots/channels
    bf = w.block[0]
    slab = np.ascontiguousarray(lat[:, :, :bf])
    t = time.perf_counter(); oracle.block_scores(slab, w.block); dt = time.perf_counter() - t
    est += dt * (w.F / bf); parts.append(f"scores {bf}/{w.F} frames")
    # a2 + a3 in full
    t = time.perf_counter()
    lv = oracle.classify(field, w.frac_active, w.frac_static)
    off, idx, _ = oracle.build_schedule(lv, (w.F, w.H, w.W), w.patch, w.patch, w.T, w.warmup,
                                        w.cooldown, w.period_moderate, w.period_static)
    est += time.perf_counter() - t; parts.append("classify+schedule full")
    n_act = int(off[w.warmup + 1] - off[w.warmup])
    sel = idx[off[w.warmup]:off[w.warmup + 1]]
    # a4 on 256 rows, in place
    m = min(256, n_act)
    t = time.perf_counter()
    oracle.kv_scatter(bits["ka"][:m], bits["va"][:m], sel[:m], bits["kb"], bits["vb"], inplace=True)
    dt = time.perf_counter() - t
    est += dt * n_act / m; parts.append(f"scatter {m} rows")
    # a5 on budget_rows rows x all heads x all keys
    g = np.random.default_rng(rng_seed)
    rows = np.sort(g.choice(n_act, size=min(budget_rows, n_act), replace=False)).astype(np.int32)
    t = time.perf_counter(); oracle.active_attention(bits["qb"], bits["kb"], bits["vb"], rows=rows)
    dt = time.perf_counter() - t
    est += dt * n_act / rows.size; parts.append(f"attention {rows.size} rows x {H} heads x {N} keys")
    flops = 4.0 * n_act * N * d * H
    return est, flops, "; ".join(parts) + " (single-threaded fp64 C, extrapolated per stage)"


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
    analyzer reads all K+1.  A plain torch.sum over the analyzer's bytes,
    timed the same way, gives the rate a single pass of that size reaches."""
    import torch
    K, C = hp.K, hp.C
    x = hp.lat[K]
    out = torch.empty_like(hp.scores)
    geom = hp.lg.c()
    flush = torch.ones(64 << 20, dtype=torch.float32, device=hp.dev)
    snap_bytes = float(x.numel()) * 4 + out.numel() * 4
    lat_bytes = float(hp.lat.numel()) * 4 + out.numel() * 4
    ops = {
        "fft_score": (lambda: J.jano_fft_scores(x, C, geom, cutoff, out, stream), snap_bytes),
        "block_scores_same_conditions": (lambda: J.jano_block_scores(hp.lat, K, C, geom, hp.w_t, hp.w_s,
                                                                     out, stream), lat_bytes),
        "plain_read_same_bytes": (lambda: torch.sum(hp.lat), float(hp.lat.numel()) * 4),
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
    code = J.device_error(stream)
    if code:
        raise RuntimeError(f"device error in the FFT score: {J.jano_status_str(code)}")
    return res


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    inp, k_cache, v_cache, n_cap = make_inputs(w)
    bits = oracle_inputs(inp, k_cache, v_cache, n_cap)
    # attention rows per step: the bounded sample shrinks with the step count
    # so that the whole run stays within a few minutes (about 2.3 s per row)
    rows = args.ref_rows if args.ref_rows > 0 else max(1, min(8, 60 // max(1, args.steps + args.warmup)))
    times = []
    flops = None
    sample = ""
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        est, flops, sample = cpu_oracle_step_time(w, inp, bits, budget_rows=rows, rng_seed=i)
        if i >= args.warmup:
            times.append(est)
        log(f"reference step {i}: estimated full step {est:.1f} s (wall {time.perf_counter()-t0:.1f} s)")
    t = statistics.mean(times)
    value = flops / t / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
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
    kernels["active_attention"]["frac_of_burst_peak"] = att_tflops / pk["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": att_tflops, "peak": bf16_sus, "unit": "TFLOP/s",
                "frac": att_tflops / bf16_sus,
                "traffic": traffic_for("kv_cache_analyzer_b200/csrc/attention.cu", w.name),
                "peak_kind": f"{pk_src} sustained cuBLAS bf16 (kernel timed inside a long step)",
                "kernel": "active_attention"}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        t0 = time.perf_counter()
        bits = oracle_inputs(inp, k_cache, v_cache, n_cap)
        est, fl, sample = cpu_oracle_step_time(w, inp, bits, budget_rows=args.ref_rows if args.ref_rows > 0 else 8)
        cpu = {"value": fl / est / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": sample, "wall_s": time.perf_counter() - t0}

    next_rows = None
    if not args.no_next:
        next_rows = measure_projections(J, hp, step, stream, pk,
                                        cpu_rows=0 if args.no_cpu_baseline or world > 1 else 2)
        next_rows.update(measure_fft_score(J, hp, stream, pk))
        next_rows.update(measure_attention_sizes(J, hp, stream, pk))

    cfg = workload_config(w)
    cache_gb = 2.0 * w.n_tokens * w.heads * w.d * 2 / 1e9
    act_gb = 3.0 * n_cap * w.heads * w.d * 2 / 1e9
    cfg.update({"n_active": n_act, "global_batch": world, "parallelism": f"replicas x{world}",
                "l2": f"no flush: the per-step working set (K/V cache {cache_gb:.2f} GB, Q/K/V act "
                      f"{act_gb:.2f} GB) is larger than the 126 MB L2"})
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": (KERNELS_PER_STEP + (1 if hp.last_split > 1 else 0)) * args.steps, "clocks": clk.summary(),
            "kernels": kernels, "next_rows": next_rows,
            "peaks": {"source": pk_src, "hbm_gbs": hbm,
                                          "bf16_tflops": pk["bf16_tflops"],
                                          "bf16_tflops_sustained": bf16_sus}}
    print(json.dumps(line), flush=True)
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
                    help="attention rows per oracle sample (0: 8 for the GPU arm's baseline, "
                         "sized from --steps/--warmup for --impl reference)")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the projections measured beside the step")
    args = ap.parse_args()

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
