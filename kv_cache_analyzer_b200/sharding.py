"""One generation of the hot path sharded over the GPUs of one node.

Attention and the KV scatter are independent per head, and the block scores
are independent per block, so rank r of W takes

* the heads [head_range(r)) of the KV cache, of the due tokens' Q/K/V and of
  the attention output (its own [N][H_r][d] tensors, no exchange), and
* the frame-blocks [frame_block_range(r)) of the analyzer: the latent frames
  of those blocks plus one halo frame (the f+1 neighbours of the last block),
  scored in place, then one all-gather puts every rank's block scores in
  frame-block order on every rank.

The level split and the schedule are then computed redundantly on every rank
(deterministic, so identical), and every rank runs scatter and attention on
its heads.  The all-gather is the only exchange of the step (77 KB of fp32
scores for the large video latent); it is a callable so that the collective
is torch.distributed's (NCCL on the GPUs) in production and any equivalent in
a test.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import (Geometry, Schedule, SplitWorkspace, attention_auto, jano_block_scores,
               jano_build_schedule, jano_build_schedule_workspace_bytes, jano_classify,
               jano_kv_scatter)


def head_range(rank: int, world: int, heads: int) -> tuple[int, int]:
    """Contiguous heads of `rank` (the first heads % world ranks take one more)."""
    return rank * heads // world, (rank + 1) * heads // world


def frame_block_range(rank: int, world: int, n_fb: int) -> tuple[int, int]:
    """Contiguous frame-blocks of `rank`."""
    return rank * n_fb // world, (rank + 1) * n_fb // world


def slab_frames(rank: int, world: int, F: int, bf: int) -> tuple[int, int, int]:
    """(first frame, frames owned, frames in the slab incl. the halo frame);
    a rank that owns no frame-block gets an empty slab."""
    n_fb = -(-F // bf)
    lo, hi = frame_block_range(rank, world, n_fb)
    f0, f1 = lo * bf, min(hi * bf, F)
    if f1 == f0:
        return f0, 0, 0
    halo = 1 if f1 < F else 0
    return f0, f1 - f0, f1 - f0 + halo


def torch_all_gather(local: torch.Tensor, full: torch.Tensor, counts: list[int]):
    """All-gather of every rank's block scores into `full` (rank order) with
    torch.distributed.  Ranks may own different numbers of blocks: the
    exchange then uses rows padded to the largest count."""
    import torch.distributed as dist
    m = max(counts)
    if all(c == m for c in counts):
        dist.all_gather_into_tensor(full, local)
        return
    pad = torch.zeros(m, dtype=local.dtype, device=local.device)
    pad[:local.numel()].copy_(local)
    buf = torch.empty(len(counts) * m, dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(buf, pad)
    o = 0
    for r, c in enumerate(counts):
        full[o:o + c].copy_(buf[r * m:r * m + c])
        o += c


class ShardedHotPath:
    """This rank's share of one sampling step (see the module docstring).

    Buffers: `lat` is the rank's latent slab [K+1][C][F_slab][H][W];
    `q_act`, `k_act`, `v_act` [n_cap][H_r][d] and `k_cache`, `v_cache`, `out`
    [N][H_r][d] hold the rank's heads; `scores` [n_blocks] all ranks' block
    scores after the gather."""

    def __init__(self, *, rank: int, world: int, K: int, C: int, latent_geom: Geometry,
                 token_geom: Geometry, heads: int, d: int, frac_active: float,
                 frac_static: float, sched: Schedule, device="cuda",
                 stream: Optional[torch.cuda.Stream] = None,
                 all_gather: Callable = torch_all_gather,
                 w_temporal: float = 0.5, w_spatial: float = 0.5):
        self.rank, self.world = rank, world
        self.K, self.C, self.d = K, C, d
        self.lg, self.tg, self.sched = latent_geom, token_geom, sched
        self.frac_active, self.frac_static = frac_active, frac_static
        self.w_t, self.w_s = w_temporal, w_spatial
        self.all_gather = all_gather
        self.dev = torch.device(device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.dev)
        e = dict(device=self.dev)
        lg = latent_geom
        bf, bh, bw = lg.block
        self.h_lo, self.h_hi = head_range(rank, world, heads)
        self.heads = self.h_hi - self.h_lo
        self.f0, self.f_own, self.f_slab = slab_frames(rank, world, lg.F, bf)
        self.slab_geom = Geometry(self.f_slab, lg.H, lg.W, lg.block, lg.patch)
        n_fb = -(-lg.F // bf)
        per_fb = (-(-lg.H // bh)) * (-(-lg.W // bw))
        self.counts = [(frame_block_range(r, world, n_fb)[1] - frame_block_range(r, world, n_fb)[0]) * per_fb
                       for r in range(world)]
        self.n_local = self.counts[rank]
        self.lat = torch.empty((K + 1, C, self.f_slab, lg.H, lg.W), dtype=torch.float32, **e)
        self.slab_scores = torch.empty(self.slab_geom.n_blocks, dtype=torch.float32, **e)
        self.scores = torch.empty(lg.n_blocks, dtype=torch.float32, **e)
        N = token_geom.n_tokens
        self.N = N
        self.field = torch.empty(token_geom.n_blocks, dtype=torch.float32, **e)
        self.levels = torch.empty(token_geom.n_blocks, dtype=torch.uint8, **e)
        self.offsets = torch.empty(sched.T + 1, dtype=torch.int32, **e)
        self.idx = torch.empty(sched.T * N, dtype=torch.int32, **e)
        self.token_levels = torch.empty(N, dtype=torch.uint8, **e)
        self.ws_bytes = jano_build_schedule_workspace_bytes(token_geom.c())
        self.ws = torch.empty(max(16, self.ws_bytes), dtype=torch.uint8, **e)
        shape = (N, self.heads, d)
        self.k_cache = torch.empty(shape, dtype=torch.bfloat16, **e)
        self.v_cache = torch.empty(shape, dtype=torch.bfloat16, **e)
        self.out = torch.zeros(shape, dtype=torch.bfloat16, **e)
        self.att_ws = SplitWorkspace(self.dev)   # key-split attention workspace
        self.last_split = 1
        self.q_act = self.k_act = self.v_act = None
        self.host_offsets = None
        self._sgc, self._tgc, self._sc = self.slab_geom.c(), token_geom.c(), sched.c()

    # ------------------------------------------------------------------ data
    def set_activations(self, n_act_cap: int):
        e = dict(device=self.dev, dtype=torch.bfloat16)
        shape = (n_act_cap, self.heads, self.d)
        self.q_act, self.k_act, self.v_act = (torch.empty(shape, **e) for _ in range(3))

    def load_latent(self, lat_full: torch.Tensor):
        """This rank's frames (and the halo frame) of the full latent history."""
        with torch.cuda.stream(self.stream):
            self.lat.copy_(lat_full[:, :, self.f0:self.f0 + self.f_slab])

    def head_slice(self, t: torch.Tensor) -> torch.Tensor:
        """This rank's heads of a [rows][heads][d] tensor."""
        return t[:, self.h_lo:self.h_hi]

    # ------------------------------------------------------------------ step
    def run_local_scores(self):
        """a1 on this rank's slab (its own blocks first, the halo frame's last);
        nothing when the rank owns no frame-block (more ranks than blocks)."""
        if self.n_local:
            jano_block_scores(self.lat, self.K, self.C, self._sgc, self.w_t, self.w_s,
                              self.slab_scores, self.stream)

    def local_scores(self) -> torch.Tensor:
        return self.slab_scores[:self.n_local]

    def run_after_gather(self):
        """a2, a3 (the same on every rank)."""
        s = self.stream
        jano_classify(self.field, self.field.numel(), self.frac_active, self.frac_static,
                      self.levels, s)
        jano_build_schedule(self.levels, self._tgc, self._sc, self.offsets, self.idx,
                            self.idx.numel(), self.token_levels, self.ws, self.ws_bytes, s)

    def run_plan_kernels(self):
        self.run_local_scores()
        with torch.cuda.stream(self.stream):
            self.all_gather(self.local_scores(), self.scores, self.counts)
        self.run_after_gather()

    def plan(self):
        self.run_plan_kernels()
        # the copy is ordered after the kernels on their own stream
        with torch.cuda.stream(self.stream):
            self.host_offsets = self.offsets.to("cpu", non_blocking=False).tolist()
        return self.host_offsets

    def due(self, step: int):
        o = self.host_offsets
        return o[step], o[step + 1] - o[step]

    def run_head_kernels(self, step: int):
        """a4, a5 of sampling step `step` on this rank's heads (none when the
        rank owns no head: more ranks than heads)."""
        s = self.stream
        start, n_act = self.due(step)
        if self.heads == 0:
            return n_act
        idx = self.idx[start:start + n_act]
        jano_kv_scatter(self.k_act, self.v_act, idx, n_act, self.heads, self.d,
                        self.k_cache, self.v_cache, self.N, s)
        # a rank's few heads give few CTAs: the keys are split when that fills the SMs better
        self.last_split = attention_auto(self.q_act, self.k_cache, self.v_cache, idx, n_act, self.N,
                                         self.heads, self.d, self.out, s, self.att_ws)
        return n_act

    def run_step_kernels(self, step: int):
        """a1..a5 of sampling step `step` for this rank's blocks and heads."""
        self.run_plan_kernels()
        return self.run_head_kernels(step)
