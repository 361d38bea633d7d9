"""Per-workload test inputs: seeded tensors from ``synth`` plus the oracle's
level maps and index lists (the GPU path computes its own and they are
compared bit for bit; where a GPU kernel needs an index list as input, the
test hands it the oracle's so both sides see identical inputs)."""
from __future__ import annotations

import functools
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle
import synth


def token_field(w: synth.Workload) -> np.ndarray:
    TF, TH, TW = w.grid
    return synth.token_field(TF, TH, TW, seed=w.seed * 10 + 1, sigma=w.field_sigma)


def token_geometry(w: synth.Workload):
    """Geometry in which every token is its own block (the per-token field)."""
    return (w.F, w.H, w.W), w.patch, w.patch


@functools.lru_cache(maxsize=2)
def attention_case(name: str):
    """Inputs of one active-only attention step of workload `name`."""
    w = synth.WORKLOADS[name]
    N, H, d = w.n_tokens, w.heads, w.d
    field = token_field(w)
    levels = oracle.classify(field, w.frac_active, w.frac_static)
    dims, block, patch = token_geometry(w)
    off, idx_all, _ = oracle.build_schedule(levels, dims, block, patch, w.T, w.warmup,
                                            w.cooldown, w.period_moderate, w.period_static)
    s = w.warmup                      # first interleaved step: Active tokens only
    idx = idx_all[off[s]:off[s + 1]].copy()
    base = w.seed * 1000
    q_act = synth.normal_bf16((idx.size, H, d), base + 1)
    k_fresh = synth.normal_bf16((N, H, d), base + 2)
    v_fresh = synth.normal_bf16((N, H, d), base + 3)
    k_stale = synth.perturb_bf16(k_fresh, 0.05, base + 4)
    v_stale = synth.perturb_bf16(v_fresh, 0.05, base + 5)
    return dict(w=w, field=field, levels=levels, idx=idx, q_act=q_act,
                k_act=k_fresh[idx].contiguous(), v_act=v_fresh[idx].contiguous(),
                k_stale=k_stale, v_stale=v_stale)


@functools.lru_cache(maxsize=2)
def latent(name: str) -> np.ndarray:
    w = synth.WORKLOADS[name]
    return synth.latent_history(w.K, w.C, w.F, w.H, w.W, seed=w.seed)


def sample_rows(n_act: int, k: int, seed: int) -> np.ndarray:
    """First, last and k-2 seeded random active rows (covers both tails)."""
    if n_act <= k:
        return np.arange(n_act, dtype=np.int32)
    g = np.random.default_rng(seed)
    mid = g.choice(np.arange(1, n_act - 1), size=k - 2, replace=False)
    return np.unique(np.concatenate([[0, n_act - 1], mid])).astype(np.int32)


def attention_errors(gpu: np.ndarray, ref: np.ndarray):
    """(max-abs, mean-rel = sum|gpu-ref| / sum|ref|) over all elements."""
    diff = np.abs(gpu.astype(np.float64) - ref)
    return float(diff.max()), float(diff.sum() / np.abs(ref).sum())


# ------------------------------------------------------------------ oracle in parallel
def _pool_workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_attention_rows(q_bits, k_bits, v_bits, rows, scale=None, chunk=4):
    """oracle.active_attention for the given active rows, the rows cut into
    chunks that run concurrently on the host cores (the oracle is a C call
    made through ctypes, which releases the GIL; each call is the unchanged
    single-threaded oracle on its own rows)."""
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    parts = [rows[i:i + chunk] for i in range(0, rows.size, chunk)]
    with ThreadPoolExecutor(max_workers=_pool_workers()) as ex:
        outs = list(ex.map(lambda r: oracle.active_attention(q_bits, k_bits, v_bits, scale=scale,
                                                             rows=r), parts))
    return np.concatenate(outs, axis=0)


def oracle_gemm_rows(x_bits, w_bits, src_rows, chunk=2):
    """oracle.gather_gemm for the given source rows, chunks run concurrently
    on the host cores (as oracle_attention_rows)."""
    src_rows = np.ascontiguousarray(src_rows, dtype=np.int32)
    parts = [src_rows[i:i + chunk] for i in range(0, src_rows.size, chunk)]
    with ThreadPoolExecutor(max_workers=_pool_workers()) as ex:
        outs = list(ex.map(lambda r: oracle.gather_gemm(x_bits, w_bits, r), parts))
    return np.concatenate(outs, axis=0)


def cta_position_rows(n_act: int, n_ctas: int = 32, seed: int = 0, tile: int = 128,
                      pair: int = 2, lanes: int = 32) -> np.ndarray:
    """Active rows that reach every position of the attention kernel's grid:
    for a spread of CTAs (first, last and evenly spaced ones between), one
    row in each (query tile of the CTA's pair, 32-row TMEM lane quarter),
    at a seeded lane; rows past n_act (the ragged last pair) are replaced by
    the last rows that exist.  Row 0 and row n_act - 1 are always included."""
    g = np.random.default_rng(seed)
    per_cta = tile * pair
    total = -(-n_act // per_cta)
    ctas = np.unique(np.linspace(0, total - 1, min(n_ctas, total)).round().astype(int))
    rows = [0, n_act - 1]
    for c in ctas:
        for t in range(pair):
            for q in range(tile // lanes):
                r = c * per_cta + t * tile + q * lanes + int(g.integers(lanes))
                rows.append(r if r < n_act else n_act - 1 - int(g.integers(min(lanes, n_act))))
    return np.unique(np.array(rows, dtype=np.int32))
