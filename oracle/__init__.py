"""fp64 CPU oracle for the Jano hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``kv_cache_analyzer_b200``) never imports, links or calls it, and this
package never imports the product library: the two share only the seeded
input generators in ``synth``.

The arithmetic lives in ``jano_oracle.c`` (plain C, fp64); this module
compiles it with gcc on first use and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "jano_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libjano_oracle.so")
_lib = None

OK, EINVAL, ESHAPE, ENONFINITE, EINDEX = 0, 1, 2, 5, 6


class OracleError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, IEEE fp64, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = C.CDLL(build())
        P = C.c_void_p
        i, d, f, ll = C.c_int, C.c_double, C.c_float, C.c_longlong
        lib.oracle_block_scores.argtypes = [P, i, i, i, i, i, i, i, i, d, d, P]
        lib.oracle_block_scores_literal.argtypes = [P, i, i, i, i, i, i, i, i, d, d, P]
        lib.oracle_level_counts.argtypes = [i, f, f, P, P]
        lib.oracle_classify.argtypes = [P, i, f, f, P]
        lib.oracle_build_schedule.argtypes = [P, i, i, i, i, i, i, i, i, i,
                                              i, i, i, i, i, P, P, ll, P]
        lib.oracle_kv_scatter.argtypes = [P, P, P, i, i, P, P, i]
        lib.oracle_active_attention.argtypes = [P, P, P, i, i, i, i, d, P, i, P]
        lib.oracle_gather_gemm.argtypes = [P, i, P, i, P, i, i, P]
        lib.oracle_splitmix64.argtypes = [C.c_uint64, i, P]
        lib.oracle_splitmix64.restype = None
        lib.oracle_random_scores.argtypes = [i, C.c_uint64, P]
        lib.oracle_fft_scores.argtypes = [P, i, i, i, i, i, i, i, i, P]
        for fn in ("oracle_block_scores", "oracle_block_scores_literal", "oracle_level_counts", "oracle_classify",
                   "oracle_build_schedule", "oracle_kv_scatter", "oracle_active_attention",
                   "oracle_gather_gemm", "oracle_random_scores", "oracle_fft_scores"):
            getattr(lib, fn).restype = C.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _check(fn, code):
    if code != OK:
        raise OracleError(fn, code)


def block_scores(lat, block, w_temporal=0.5, w_spatial=0.5):
    """lat fp32 [K+1][C][F][H][W] -> fp64 scores [nBf*nBh*nBw]."""
    lat = np.ascontiguousarray(lat, dtype=np.float32)
    K1, Cc, F, H, W = lat.shape
    bf, bh, bw = block
    nB = (-(-F // bf)) * (-(-H // bh)) * (-(-W // bw))
    out = np.empty(nB, dtype=np.float64)
    _check("oracle_block_scores", _load().oracle_block_scores(
        _ptr(lat), K1 - 1, Cc, F, H, W, bf, bh, bw, w_temporal, w_spatial, _ptr(out)))
    return out


def block_scores_literal(lat, block, w_temporal=0.5, w_spatial=0.5):
    """The literal reading: second differences over the steps of the temporal
    and spatial gradients.  lat fp32 [K+1][C][F][H][W] -> fp64 scores."""
    lat = np.ascontiguousarray(lat, dtype=np.float32)
    K1, Cc, F, H, W = lat.shape
    bf, bh, bw = block
    nB = (-(-F // bf)) * (-(-H // bh)) * (-(-W // bw))
    out = np.empty(nB, dtype=np.float64)
    _check("oracle_block_scores_literal", _load().oracle_block_scores_literal(
        _ptr(lat), K1 - 1, Cc, F, H, W, bf, bh, bw, w_temporal, w_spatial, _ptr(out)))
    return out


def level_counts(B, frac_active, frac_static):
    a, s = C.c_longlong(), C.c_longlong()
    _check("oracle_level_counts", _load().oracle_level_counts(
        B, frac_active, frac_static, C.byref(a), C.byref(s)))
    return a.value, s.value


def classify(scores_f32, frac_active, frac_static):
    """fp32 scores [B] -> uint8 levels [B] in {1,2,3}."""
    s = np.ascontiguousarray(scores_f32, dtype=np.float32)
    out = np.empty(s.shape[0], dtype=np.uint8)
    _check("oracle_classify", _load().oracle_classify(
        _ptr(s), s.shape[0], frac_active, frac_static, _ptr(out)))
    return out


def build_schedule(block_levels, dims, block, patch, T, warmup, cooldown,
                   period_moderate, period_static):
    """-> (offsets int32 [T+1], idx int32 [offsets[T]], token_levels uint8 [NT])."""
    bl = np.ascontiguousarray(block_levels, dtype=np.uint8)
    F, H, W = dims
    pf, ph, pw = patch
    NT = (F // pf) * (H // ph) * (W // pw)
    offsets = np.empty(T + 1, dtype=np.int32)
    idx = np.empty(max(1, NT * T), dtype=np.int32)
    tl = np.empty(NT, dtype=np.uint8)
    _check("oracle_build_schedule", _load().oracle_build_schedule(
        _ptr(bl), F, H, W, *block, *patch, T, warmup, cooldown,
        period_moderate, period_static, _ptr(offsets), _ptr(idx), NT * T, _ptr(tl)))
    return offsets, idx[: offsets[T]].copy(), tl


def kv_scatter(k_act, v_act, idx, k_cache, v_cache, inplace=False):
    """Returns the updated (k_cache, v_cache) uint16 arrays: copies of the
    inputs, or (inplace=True, C-contiguous uint16 caches) the caches themselves."""
    k_act = np.ascontiguousarray(k_act, dtype=np.uint16)
    v_act = np.ascontiguousarray(v_act, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    if inplace:
        assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
        assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
        kc, vc = k_cache, v_cache
    else:
        kc = np.array(k_cache, dtype=np.uint16, copy=True, order="C")
        vc = np.array(v_cache, dtype=np.uint16, copy=True, order="C")
    n_tokens = kc.shape[0]
    row = int(np.prod(kc.shape[1:]))
    _check("oracle_kv_scatter", _load().oracle_kv_scatter(
        _ptr(k_act), _ptr(v_act), _ptr(idx), idx.shape[0], row, _ptr(kc), _ptr(vc), n_tokens))
    return kc, vc


def active_attention(q_act, k_cache, v_cache, scale=None, rows=None):
    """BF16 bits q_act [n_act][heads][d], caches [N][heads][d] ->
    fp64 [len(rows)][heads][d] for the requested active rows (default: all)."""
    q = np.ascontiguousarray(q_act, dtype=np.uint16)
    kc = np.ascontiguousarray(k_cache, dtype=np.uint16)
    vc = np.ascontiguousarray(v_cache, dtype=np.uint16)
    n_act, heads, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows = np.arange(n_act, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    out = np.empty((rows.shape[0], heads, d), dtype=np.float64)
    _check("oracle_active_attention", _load().oracle_active_attention(
        _ptr(q), _ptr(kc), _ptr(vc), n_act, kc.shape[0], heads, d, float(scale),
        _ptr(rows), rows.shape[0], _ptr(out)))
    return out


def gather_gemm(x, w, gather=None):
    """BF16 bits x [n_x][k], w [n][k], optional int32 gather [m] ->
    fp64 [m][n] with out[r] = x[gather[r]] @ w^T (x[r] without gather)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    n_x, k = x.shape
    n = w.shape[0]
    assert w.shape[1] == k
    g = None if gather is None else np.ascontiguousarray(gather, dtype=np.int32)
    m = n_x if g is None else g.shape[0]
    out = np.empty((m, n), dtype=np.float64)
    _check("oracle_gather_gemm", _load().oracle_gather_gemm(
        _ptr(x), n_x, _ptr(g), m, _ptr(w), n, k, _ptr(out)))
    return out


def splitmix64(seed, n):
    """The first n outputs of splitmix64 seeded with `seed` (uint64)."""
    out = np.empty(n, dtype=np.uint64)
    _load().oracle_splitmix64(C.c_uint64(seed), n, _ptr(out))
    return out


def fft_scores(x, block, cutoff):
    """High-band spectral energy per block of one snapshot.
    x fp32 [C][F][H][W] -> fp64 scores [nBf*nBh*nBw]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    Cc, F, H, W = x.shape
    bf, bh, bw = block
    nB = (-(-F // bf)) * (-(-H // bh)) * (-(-W // bw))
    out = np.empty(nB, dtype=np.float64)
    _check("oracle_fft_scores", _load().oracle_fft_scores(_ptr(x), Cc, F, H, W, bf, bh, bw, cutoff,
                                                          _ptr(out)))
    return out


def random_scores(n, seed):
    """Uniform [0, 1) fp32 scores of the random-masking ablation (24 bits)."""
    out = np.empty(n, dtype=np.float32)
    _check("oracle_random_scores", _load().oracle_random_scores(n, C.c_uint64(seed), _ptr(out)))
    return out
