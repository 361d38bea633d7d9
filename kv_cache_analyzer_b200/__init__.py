"""kv_cache_analyzer_b200 -- Python binding of libjano, the B200 (sm_100a)
library for the data-parallel hot path of Jano (block-wise complexity
analyzer, three-level token schedule, KV-cache scatter and active-query
attention).

The functions named ``jano_*`` mirror the C ABI in ``include/jano.h`` one to
one: they only marshal torch tensors (device memory) and the current CUDA
stream into the C call and turn a non-OK status into ``JanoError``.  The
lower-case helpers below them allocate outputs with torch and call those.
Every step of the path runs in the library's CUDA kernels; there is no CPU
or PyTorch fallback, and importing a function fails loudly when the library
is not built.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

__all__ = [
    "JanoError", "jano_geom", "jano_sched_cfg", "lib", "library_path",
    "jano_block_scores", "jano_classify", "jano_build_schedule_workspace_bytes",
    "jano_build_schedule", "jano_build_schedule_noalloc", "jano_kv_scatter", "jano_active_attention",
    "jano_active_attention_split", "jano_active_attention_workspace_bytes", "jano_active_attention_splits",
    "jano_active_attention_splits_on", "jano_get_device_error", "jano_status_str", "jano_version",
    "Geometry", "Schedule", "block_scores", "classify", "build_schedule",
    "kv_scatter", "active_attention", "device_error",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# JANO_LIBRARY may point at another build of the same library (e.g. a
# variant compiled with different tuning macros).
library_path = os.environ.get("JANO_LIBRARY") or os.path.join(_HERE, "libjano.so")

STATUS_NAMES = {0: "JANO_OK", 1: "JANO_EINVAL", 2: "JANO_ESHAPE", 3: "JANO_EALIGN",
                4: "JANO_EUNSUPPORTED", 5: "JANO_ENONFINITE", 6: "JANO_EINDEX",
                7: "JANO_ETIMEOUT", 8: "JANO_ECUDA"}
EXPORTS = ("jano_block_scores", "jano_block_scores_literal", "jano_classify", "jano_build_schedule_workspace_bytes",
           "jano_build_schedule", "jano_build_schedule_noalloc", "jano_kv_scatter", "jano_active_attention",
           "jano_active_attention_split", "jano_active_attention_workspace_bytes", "jano_active_attention_splits",
           "jano_active_attention_splits_on", "jano_gather_gemm", "jano_qkv_project", "jano_random_scores", "jano_fft_scores",
           "jano_stream_sum", "jano_get_device_error", "jano_status_str", "jano_version")


class JanoError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


class jano_geom(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("F", "H", "W", "bf", "bh", "bw", "pf", "ph", "pw")]


class jano_sched_cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("T", "warmup", "cooldown", "period_moderate", "period_static")]


_lib = None


def lib() -> C.CDLL:
    """Load libjano.so (built in-tree by ``python -m kv_cache_analyzer_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"libjano.so is not built at {library_path}; "
                               "run `python -m kv_cache_analyzer_b200.build`")
        L = C.CDLL(library_path)
        P, i, f, z = C.c_void_p, C.c_int, C.c_float, C.c_size_t
        G, S = C.POINTER(jano_geom), C.POINTER(jano_sched_cfg)
        L.jano_block_scores.argtypes = [P, i, i, G, f, f, P, P]
        L.jano_block_scores_literal.argtypes = [P, i, i, G, f, f, P, P]
        L.jano_classify.argtypes = [P, i, f, f, P, P]
        L.jano_build_schedule_workspace_bytes.argtypes = [G]
        L.jano_build_schedule_workspace_bytes.restype = z
        L.jano_build_schedule.argtypes = [P, G, S, P, P, z, P, P, z, P]
        L.jano_build_schedule_noalloc.argtypes = [P, G, S, P, P, z, P, P]
        L.jano_kv_scatter.argtypes = [P, P, P, i, i, i, P, P, i, P]
        L.jano_active_attention.argtypes = [P, P, P, P, i, i, i, i, f, P, P]
        L.jano_active_attention_split.argtypes = [P, P, P, P, i, i, i, i, f, i, P, z, P, P]
        L.jano_active_attention_workspace_bytes.argtypes = [i, i, i, i]
        L.jano_active_attention_workspace_bytes.restype = z
        L.jano_active_attention_splits.argtypes = [i, i, i, i]
        L.jano_active_attention_splits.restype = C.c_int
        L.jano_active_attention_splits_on.argtypes = [i, i, i, i, i]
        L.jano_active_attention_splits_on.restype = C.c_int
        L.jano_gather_gemm.argtypes = [P, i, P, i, P, i, i, P, P, i, P]
        L.jano_qkv_project.argtypes = [P, i, P, i, P, i, i, P, P, P, P]
        L.jano_random_scores.argtypes = [i, C.c_uint64, P, P]
        L.jano_fft_scores.argtypes = [P, i, G, i, P, P]
        L.jano_stream_sum.argtypes = [P, C.c_longlong, P, i, P]
        L.jano_get_device_error.argtypes = [P]
        L.jano_status_str.argtypes = [i]
        L.jano_status_str.restype = C.c_char_p
        L.jano_version.argtypes = []
        for fn in ("jano_block_scores", "jano_block_scores_literal", "jano_classify", "jano_build_schedule",
                   "jano_build_schedule_noalloc", "jano_kv_scatter", "jano_active_attention",
                   "jano_active_attention_split", "jano_get_device_error",
                   "jano_gather_gemm", "jano_qkv_project", "jano_random_scores", "jano_fft_scores",
                   "jano_stream_sum", "jano_version"):
            getattr(L, fn).restype = C.c_int
        _lib = L
    return _lib


def _torch_stream(stream):
    """The torch stream object for `stream` (None: the current stream; a raw
    cudaStream_t handle is wrapped), for allocator bookkeeping."""
    if stream is None:
        return torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream))


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t: torch.Tensor | None, name: str, dtype=None) -> C.c_void_p | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return C.c_void_p(t.data_ptr())


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise JanoError(fn, code)


# ---------------------------------------------------------------- C ABI mirror
def jano_block_scores(lat, K, C_, geom, w_temporal, w_spatial, scores, stream=None):
    _check("jano_block_scores", lib().jano_block_scores(
        _dev(lat, "lat", torch.float32), K, C_, C.byref(geom), w_temporal, w_spatial,
        _dev(scores, "scores", torch.float32), _stream(stream)))


def jano_block_scores_literal(lat, K, C_, geom, w_temporal, w_spatial, scores, stream=None):
    _check("jano_block_scores_literal", lib().jano_block_scores_literal(
        _dev(lat, "lat", torch.float32), K, C_, C.byref(geom), w_temporal, w_spatial,
        _dev(scores, "scores", torch.float32), _stream(stream)))


def jano_classify(scores, n_blocks, frac_active, frac_static, levels, stream=None):
    _check("jano_classify", lib().jano_classify(
        _dev(scores, "scores", torch.float32), n_blocks, frac_active, frac_static,
        _dev(levels, "levels", torch.uint8), _stream(stream)))


def jano_build_schedule_workspace_bytes(geom) -> int:
    return int(lib().jano_build_schedule_workspace_bytes(C.byref(geom)))


def jano_build_schedule(block_levels, geom, cfg, offsets, idx, idx_capacity, token_levels,
                        workspace, ws_bytes, stream=None):
    _check("jano_build_schedule", lib().jano_build_schedule(
        _dev(block_levels, "block_levels", torch.uint8), C.byref(geom), C.byref(cfg),
        _dev(offsets, "offsets", torch.int32), _dev(idx, "idx", torch.int32), idx_capacity,
        _dev(token_levels, "token_levels", torch.uint8), _dev(workspace, "workspace"),
        ws_bytes, _stream(stream)))


def jano_build_schedule_noalloc(block_levels, geom, cfg, offsets, idx, idx_capacity, token_levels,
                                stream=None):
    """jano_build_schedule without a workspace argument: for callers that
    cannot allocate device memory.  The library's own 1 MiB device array
    serves as scratch (geometries of at most 1,036,416 tokens); calls
    overlapping on the GPU race on it, and the first call on a device should
    come before any stream capture."""
    _check("jano_build_schedule_noalloc", lib().jano_build_schedule_noalloc(
        _dev(block_levels, "block_levels", torch.uint8), C.byref(geom), C.byref(cfg),
        _dev(offsets, "offsets", torch.int32), _dev(idx, "idx", torch.int32), idx_capacity,
        _dev(token_levels, "token_levels", torch.uint8), _stream(stream)))


def jano_kv_scatter(k_act, v_act, idx, n_act, heads, d, k_cache, v_cache, n_tokens, stream=None):
    _check("jano_kv_scatter", lib().jano_kv_scatter(
        _dev(k_act, "k_act", torch.bfloat16), _dev(v_act, "v_act", torch.bfloat16),
        _dev(idx, "idx", torch.int32), n_act, heads, d,
        _dev(k_cache, "k_cache", torch.bfloat16), _dev(v_cache, "v_cache", torch.bfloat16),
        n_tokens, _stream(stream)))


def jano_active_attention(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, scale, out,
                          stream=None):
    _check("jano_active_attention", lib().jano_active_attention(
        _dev(q_act, "q_act", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
        _dev(v_cache, "v_cache", torch.bfloat16), _dev(idx, "idx", torch.int32), n_act,
        n_tokens, heads, d, scale, _dev(out, "out", torch.bfloat16), _stream(stream)))


def jano_active_attention_split(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, scale,
                                n_split, workspace, ws_bytes, out, stream=None):
    _check("jano_active_attention_split", lib().jano_active_attention_split(
        _dev(q_act, "q_act", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
        _dev(v_cache, "v_cache", torch.bfloat16), _dev(idx, "idx", torch.int32), n_act,
        n_tokens, heads, d, scale, n_split, _dev(workspace, "workspace"), ws_bytes,
        _dev(out, "out", torch.bfloat16), _stream(stream)))


def jano_active_attention_workspace_bytes(n_act, heads, d, n_split) -> int:
    return int(lib().jano_active_attention_workspace_bytes(n_act, heads, d, n_split))


def jano_active_attention_splits(n_act, n_tokens, heads, d) -> int:
    return int(lib().jano_active_attention_splits(n_act, n_tokens, heads, d))


def jano_active_attention_splits_on(n_act, n_tokens, heads, d, sm_count) -> int:
    return int(lib().jano_active_attention_splits_on(n_act, n_tokens, heads, d, sm_count))


def jano_gather_gemm(x, n_x, gather, m, w, n, k, scatter, out, n_out, stream=None):
    _check("jano_gather_gemm", lib().jano_gather_gemm(
        _dev(x, "x", torch.bfloat16), n_x, _dev(gather, "gather", torch.int32), m,
        _dev(w, "w", torch.bfloat16), n, k, _dev(scatter, "scatter", torch.int32),
        _dev(out, "out", torch.bfloat16), n_out, _stream(stream)))


def jano_qkv_project(x, n_tokens, idx, n_act, w_qkv, hd, k, q_act, k_cache, v_cache, stream=None):
    _check("jano_qkv_project", lib().jano_qkv_project(
        _dev(x, "x", torch.bfloat16), n_tokens, _dev(idx, "idx", torch.int32), n_act,
        _dev(w_qkv, "w_qkv", torch.bfloat16), hd, k, _dev(q_act, "q_act", torch.bfloat16),
        _dev(k_cache, "k_cache", torch.bfloat16), _dev(v_cache, "v_cache", torch.bfloat16),
        _stream(stream)))


def jano_random_scores(n_blocks, seed, scores, stream=None):
    _check("jano_random_scores", lib().jano_random_scores(
        n_blocks, C.c_uint64(seed), _dev(scores, "scores", torch.float32), _stream(stream)))


def jano_fft_scores(x, C_, geom, cutoff, scores, stream=None):
    _check("jano_fft_scores", lib().jano_fft_scores(
        _dev(x, "x", torch.float32), C_, geom, cutoff, _dev(scores, "scores", torch.float32),
        _stream(stream)))


def jano_stream_sum(x, n, partial, n_partial, stream=None):
    _check("jano_stream_sum", lib().jano_stream_sum(
        _dev(x, "x", torch.float32), n, _dev(partial, "partial", torch.float32), n_partial,
        _stream(stream)))


def stream_sum(x: torch.Tensor, n_partial: int | None = None, out=None, stream=None) -> torch.Tensor:
    """Partial sums of one streaming pass over the fp32 tensor x (the read-rate
    calibration the analyzer is compared with); one CTA per SM by default."""
    if n_partial is None:
        n_partial = torch.cuda.get_device_properties(x.device).multi_processor_count
    if out is None:
        out = torch.empty(n_partial, dtype=torch.float32, device=x.device)
    jano_stream_sum(x, x.numel(), out, n_partial, stream)
    return out


def jano_get_device_error(stream=None) -> int:
    return int(lib().jano_get_device_error(_stream(stream)))


def jano_status_str(code: int) -> str:
    return lib().jano_status_str(code).decode()


def jano_version() -> int:
    return int(lib().jano_version())


# ---------------------------------------------------------------- helpers
@dataclass(frozen=True)
class Geometry:
    """Latent dims, analyzer block and token patch (latent elements)."""
    F: int
    H: int
    W: int
    block: tuple = (1, 4, 4)
    patch: tuple = (1, 2, 2)

    def c(self) -> jano_geom:
        return jano_geom(self.F, self.H, self.W, *self.block, *self.patch)

    @property
    def n_blocks(self) -> int:
        bf, bh, bw = self.block
        return (-(-self.F // bf)) * (-(-self.H // bh)) * (-(-self.W // bw))

    @property
    def n_tokens(self) -> int:
        pf, ph, pw = self.patch
        return (self.F // pf) * (self.H // ph) * (self.W // pw)


@dataclass(frozen=True)
class Schedule:
    T: int = 50
    warmup: int = 5
    cooldown: int = 5
    period_moderate: int = 2
    period_static: int = 4

    def c(self) -> jano_sched_cfg:
        return jano_sched_cfg(self.T, self.warmup, self.cooldown, self.period_moderate,
                              self.period_static)


def block_scores(lat: torch.Tensor, geom: Geometry, w_temporal=0.5, w_spatial=0.5,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    K1, Cc = lat.shape[0], lat.shape[1]
    if out is None:
        out = torch.empty(geom.n_blocks, dtype=torch.float32, device=lat.device)
    jano_block_scores(lat, K1 - 1, Cc, geom.c(), w_temporal, w_spatial, out, stream)
    return out


def block_scores_literal(lat: torch.Tensor, geom: Geometry, w_temporal=0.5, w_spatial=0.5,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The literal reading: second differences over the steps of the gradients."""
    K1, Cc = lat.shape[0], lat.shape[1]
    if out is None:
        out = torch.empty(geom.n_blocks, dtype=torch.float32, device=lat.device)
    jano_block_scores_literal(lat, K1 - 1, Cc, geom.c(), w_temporal, w_spatial, out, stream)
    return out


def classify(scores: torch.Tensor, frac_active: float, frac_static: float,
             out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(scores.numel(), dtype=torch.uint8, device=scores.device)
    jano_classify(scores, scores.numel(), frac_active, frac_static, out, stream)
    return out


def build_schedule(block_levels: torch.Tensor, geom: Geometry, sched: Schedule,
                   stream=None, workspace: torch.Tensor | None = None):
    """-> (offsets int32 [T+1], idx int32 [T*N capacity], token_levels uint8 [N])."""
    dev = block_levels.device
    g = geom.c()
    N = geom.n_tokens
    ws_bytes = jano_build_schedule_workspace_bytes(g)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    offsets = torch.empty(sched.T + 1, dtype=torch.int32, device=dev)
    idx = torch.empty(sched.T * N, dtype=torch.int32, device=dev)
    tl = torch.empty(N, dtype=torch.uint8, device=dev)
    jano_build_schedule(block_levels, g, sched.c(), offsets, idx, idx.numel(), tl, workspace,
                        workspace.numel(), stream)
    return offsets, idx, tl


def kv_scatter(k_act, v_act, idx, k_cache, v_cache, stream=None) -> None:
    n_act = idx.numel()
    N, H, d = k_cache.shape
    jano_kv_scatter(k_act, v_act, idx, n_act, H, d, k_cache, v_cache, N, stream)


def active_attention(q_act, k_cache, v_cache, idx, out, scale=None, stream=None, split=None,
                     workspace=None) -> None:
    """out[idx[i]] = attention of q_act[i] over the whole cache.  split: the
    number of key ranges per query tile (None: the library's choice for this
    shape on the current device, 1 for large due sets); with split > 1 the
    partials go to `workspace` (a device uint8 tensor of at least
    jano_active_attention_workspace_bytes bytes), allocated here if None."""
    n_act = idx.numel()
    N, H, d = k_cache.shape
    if scale is None:
        scale = d ** -0.5
    if split is None:
        split = jano_active_attention_splits(n_act, N, H, d) if n_act > 0 else 1
    if split <= 1:
        jano_active_attention(q_act, k_cache, v_cache, idx, n_act, N, H, d, scale, out, stream)
        return
    ws_bytes = jano_active_attention_workspace_bytes(n_act, H, d, split)
    temporary = workspace is None
    if temporary:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=k_cache.device)
    jano_active_attention_split(q_act, k_cache, v_cache, idx, n_act, N, H, d, scale, split,
                                workspace, workspace.numel() * workspace.element_size(), out, stream)
    if temporary:
        # freed on return: the allocator must not hand it out again before the
        # launch on `stream` has finished with it
        workspace.record_stream(_torch_stream(stream))


class SplitWorkspace:
    """Device workspaces of key-split attention, one per stream, each grown
    on demand.  Launches on one stream are ordered, so reusing that stream's
    buffer is safe; a launch on another stream gets a buffer of its own, so
    concurrent split launches never share partials."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.bufs = {}

    def get(self, nbytes: int, stream) -> torch.Tensor:
        ts = _torch_stream(stream)
        key = int(ts.cuda_stream)
        buf = self.bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            with torch.cuda.stream(ts):
                buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            self.bufs[key] = buf
        return buf


def attention_auto(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, out, stream,
                   ws: SplitWorkspace) -> int:
    """jano_active_attention, or its key-split form when the library's choice
    for this shape on this device is a split (small due sets, few heads);
    returns the split count used."""
    split = jano_active_attention_splits(n_act, n_tokens, heads, d) if n_act > 0 else 1
    if split <= 1:
        jano_active_attention(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, d ** -0.5,
                              out, stream)
        return 1
    buf = ws.get(jano_active_attention_workspace_bytes(n_act, heads, d, split), stream)
    jano_active_attention_split(q_act, k_cache, v_cache, idx, n_act, n_tokens, heads, d, d ** -0.5,
                                split, buf, buf.numel(), out, stream)
    return split


def gather_gemm(x, w, out, gather=None, scatter=None, stream=None) -> None:
    """out[scatter[r] or r] = x[gather[r] or r] @ w^T for r < m (BF16 tensors
    x [n_x][k], w [n][k], out [n_out][n]; m = len(gather or scatter or x))."""
    n_x, k = x.shape
    n = w.shape[0]
    m = gather.numel() if gather is not None else (scatter.numel() if scatter is not None else n_x)
    jano_gather_gemm(x, n_x, gather, m, w, n, k, scatter, out, out.shape[0], stream)


def qkv_project(x, idx, w_qkv, q_act, k_cache, v_cache, stream=None) -> None:
    """Q/K/V of the active tokens idx from the hidden states x [N][k]:
    q_act [n_act][hd] and the rows idx of k_cache, v_cache [N][hd] (also
    accepted as [N][heads][d])."""
    N, k = x.shape
    hd = w_qkv.shape[0] // 3
    jano_qkv_project(x, N, idx, idx.numel(), w_qkv, hd, k, q_act, k_cache, v_cache, stream)


def random_scores(n_blocks: int, seed: int, out=None, stream=None) -> torch.Tensor:
    """Uniform scores of the random-masking ablation (classify them for a
    random level map with the analyzer's level counts)."""
    if out is None:
        out = torch.empty(n_blocks, dtype=torch.float32, device="cuda")
    jano_random_scores(n_blocks, seed, out, stream)
    return out


def fft_scores(x: torch.Tensor, geom: Geometry, cutoff: int = 1, out=None, stream=None) -> torch.Tensor:
    """High-band spectral energy per block of one snapshot x [C][F][H][W]
    (the FFT baseline score)."""
    if out is None:
        out = torch.empty(geom.n_blocks, dtype=torch.float32, device=x.device)
    jano_fft_scores(x, x.shape[0], geom.c(), cutoff, out, stream)
    return out


def device_error(stream=None) -> int:
    return jano_get_device_error(stream)
