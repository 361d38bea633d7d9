"""One pass of the Jano hot path over device-resident buffers.

``HotPath`` owns the device buffers (torch allocations: plumbing only) and
runs, on one CUDA stream, the five C-ABI entry points in the order of one
sampling step of the method:

  a1  jano_block_scores     latent history      -> block scores
  a2  jano_classify         per-token field     -> token levels (Static/Moderate/Active)
  a3  jano_build_schedule   token levels        -> per-step due lists (CSR)
  a4  jano_kv_scatter       fresh K/V of the due tokens -> persistent cache
  a5  jano_active_attention due queries over the whole cache -> out[idx]
      (jano_active_attention_split for due sets too small to fill the GPU)

The CSR offsets are read back to the host once by ``plan()`` (one small
device-to-host copy per generation); ``step(s)`` then runs a1..a5 for
sampling step ``s`` with the due list of that step.  ``step_from_host``
is the same pass with the step's inputs copied in from (pinned) host memory
and the result copied back, for end-to-end timing.
"""
from __future__ import annotations

import torch

from . import (Geometry, Schedule, SplitWorkspace, attention_auto, jano_block_scores,
               jano_build_schedule, jano_build_schedule_workspace_bytes,
               jano_classify, jano_kv_scatter)

KERNELS_PER_STEP = 6      # scores 1 + classify 1 + schedule 2 + scatter 1 + attention 1
                          # (attention 2 when its keys are split: + the merge pass)


class HotPath:
    def __init__(self, *, K: int, C: int, latent_geom: Geometry, token_geom: Geometry,
                 heads: int, d: int, frac_active: float, frac_static: float,
                 sched: Schedule, device="cuda", stream: torch.cuda.Stream | None = None,
                 w_temporal: float = 0.5, w_spatial: float = 0.5):
        self.K, self.C, self.heads, self.d = K, C, heads, d
        self.lg, self.tg, self.sched = latent_geom, token_geom, sched
        self.frac_active, self.frac_static = frac_active, frac_static
        self.w_t, self.w_s = w_temporal, w_spatial
        self.dev = torch.device(device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.dev)
        N = token_geom.n_tokens
        self.N = N
        e = dict(device=self.dev)
        lg = latent_geom
        self.lat = torch.empty((K + 1, C, lg.F, lg.H, lg.W), dtype=torch.float32, **e)
        self.scores = torch.empty(lg.n_blocks, dtype=torch.float32, **e)
        self.field = torch.empty(token_geom.n_blocks, dtype=torch.float32, **e)
        self.levels = torch.empty(token_geom.n_blocks, dtype=torch.uint8, **e)
        self.offsets = torch.empty(sched.T + 1, dtype=torch.int32, **e)
        self.idx = torch.empty(sched.T * N, dtype=torch.int32, **e)
        self.token_levels = torch.empty(N, dtype=torch.uint8, **e)
        self.ws_bytes = jano_build_schedule_workspace_bytes(token_geom.c())
        self.ws = torch.empty(max(16, self.ws_bytes), dtype=torch.uint8, **e)
        self.k_cache = torch.empty((N, heads, d), dtype=torch.bfloat16, **e)
        self.v_cache = torch.empty((N, heads, d), dtype=torch.bfloat16, **e)
        self.out = torch.zeros((N, heads, d), dtype=torch.bfloat16, **e)
        self.att_ws = SplitWorkspace(self.dev)   # key-split attention workspace
        self.last_split = 1
        self.q_act = self.k_act = self.v_act = None
        self.host_offsets = None
        self._lgc, self._tgc, self._sc = lg.c(), token_geom.c(), sched.c()

    # ------------------------------------------------------------------ setup
    def set_activations(self, n_act_cap: int):
        e = dict(device=self.dev, dtype=torch.bfloat16)
        shape = (n_act_cap, self.heads, self.d)
        self.q_act = torch.empty(shape, **e)
        self.k_act = torch.empty(shape, **e)
        self.v_act = torch.empty(shape, **e)

    def run_plan_kernels(self, events=None):
        """a1..a3 on the stream (no host synchronisation)."""
        s = self.stream
        ev = events or [None] * 4
        if ev[0] is not None: ev[0].record(s)
        jano_block_scores(self.lat, self.K, self.C, self._lgc, self.w_t, self.w_s, self.scores, s)
        if ev[1] is not None: ev[1].record(s)
        jano_classify(self.field, self.field.numel(), self.frac_active, self.frac_static,
                      self.levels, s)
        if ev[2] is not None: ev[2].record(s)
        jano_build_schedule(self.levels, self._tgc, self._sc, self.offsets, self.idx,
                            self.idx.numel(), self.token_levels, self.ws, self.ws_bytes, s)
        if ev[3] is not None: ev[3].record(s)

    def use(self, bufs: dict):
        """Point the step at another set of input/output buffers (keys lat,
        field, q_act, k_act, v_act, out); the kernels take the pointers when
        they are enqueued."""
        for k, v in bufs.items():
            setattr(self, k, v)

    def plan(self):
        """Run a1..a3 once and read the CSR offsets back (one D2H per generation)."""
        self.run_plan_kernels()
        # the copy is ordered after the kernels on their own stream
        with torch.cuda.stream(self.stream):
            self.host_offsets = self.offsets.to("cpu", non_blocking=False).tolist()
        return self.host_offsets

    def due(self, step: int):
        o = self.host_offsets
        return o[step], o[step + 1] - o[step]

    # ------------------------------------------------------------------ step
    def run_step_kernels(self, step: int, events=None):
        """a1..a5 for sampling step `step`; events (6, optional) bracket the stages."""
        s = self.stream
        ev = events or [None] * 6
        self.run_plan_kernels(ev[:4])
        start, n_act = self.due(step)
        idx = self.idx[start:start + n_act]
        jano_kv_scatter(self.k_act, self.v_act, idx, n_act, self.heads, self.d,
                        self.k_cache, self.v_cache, self.N, s)
        if ev[4] is not None: ev[4].record(s)
        self.last_split = attention_auto(self.q_act, self.k_cache, self.v_cache, idx, n_act, self.N,
                                         self.heads, self.d, self.out, s, self.att_ws)
        if ev[5] is not None: ev[5].record(s)
        return n_act

    def capture_step(self, step: int) -> torch.cuda.CUDAGraph:
        """a1..a5 of sampling step `step` captured once as a CUDA graph on the
        hot path's stream (which must not be the default stream); replay()
        re-runs the step with no host launches.  One ordinary pass runs first,
        so that everything the entry points make lazily (the device error
        word, shared-memory opt-ins, the key-split workspace) exists before
        the capture."""
        self.run_step_kernels(step)
        self.stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.run_step_kernels(step)
        return g

    def capture_repeated(self, fn, times: int) -> torch.cuda.CUDAGraph:
        """`times` back-to-back calls of fn(stream) captured as one graph (the
        launch-bound plan kernels timed without per-launch host work)."""
        fn(self.stream)
        self.stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for _ in range(times):
                fn(self.stream)
        return g

    def step_from_host(self, step: int, host: dict, host_out: torch.Tensor):
        """The same pass with this step's inputs copied in from host memory
        (latent, field, q/k/v of the due tokens) and `out` copied back."""
        s = self.stream
        with torch.cuda.stream(s):
            self.lat.copy_(host["lat"], non_blocking=True)
            self.field.copy_(host["field"], non_blocking=True)
            n = host["q_act"].shape[0]
            self.q_act[:n].copy_(host["q_act"], non_blocking=True)
            self.k_act[:n].copy_(host["k_act"], non_blocking=True)
            self.v_act[:n].copy_(host["v_act"], non_blocking=True)
        self.run_step_kernels(step)
        with torch.cuda.stream(s):
            host_out.copy_(self.out, non_blocking=True)

    @staticmethod
    def h2d_bytes(host: dict) -> int:
        return sum(host[k].numel() * host[k].element_size()
                   for k in ("lat", "field", "q_act", "k_act", "v_act"))


class HostStepper:
    """End-to-end steps from pinned host memory, pipelined over three streams.

    Every step copies its inputs (latent, field, q/k/v of the due tokens) in
    from the pinned host buffers and its result (`out`) back to pinned host
    memory.  Two device sets of those buffers alternate, so the inputs of
    step i+1 are copied in (copy-in stream) and the result of step i-1 is
    copied out (copy-out stream) while step i computes on the hot path's
    stream; events order every reuse of a buffer.  The per-generation state
    (scores, levels, schedule, KV cache) stays on the compute stream."""

    IN_KEYS = ("lat", "field", "q_act", "k_act", "v_act")

    def __init__(self, hp: HotPath, host: dict, host_out: torch.Tensor):
        self.hp, self.host, self.host_out = hp, host, host_out
        dev = hp.dev
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.sets = []
        for _ in range(2):
            b = {k: torch.empty(host[k].shape, dtype=host[k].dtype, device=dev) for k in self.IN_KEYS}
            b["out"] = torch.zeros_like(hp.out)
            self.sets.append(b)
        ev = lambda: torch.cuda.Event()
        self.ev_in = [ev(), ev()]      # the set's inputs have landed
        self.ev_used = [ev(), ev()]    # the step on the set is done (inputs free, out final)
        self.ev_out = [ev(), ev()]     # the set's out is back in host memory
        self.used = [False, False]

    def _copy_in(self, b: int):
        s = self.h2d
        if self.used[b]:
            s.wait_event(self.ev_used[b])
        with torch.cuda.stream(s):
            for k in self.IN_KEYS:
                self.sets[b][k].copy_(self.host[k], non_blocking=True)
        self.ev_in[b].record(s)

    def run(self, step: int, n_steps: int, start: torch.cuda.Event | None = None,
            end: torch.cuda.Event | None = None):
        """n_steps end-to-end steps of sampling step `step`; `start` / `end`
        (optional) are recorded on the compute stream around all of them, with
        the copy streams ordered inside."""
        cs = self.hp.stream
        if start is not None:
            start.record(cs)
            self.h2d.wait_stream(cs)
            self.d2h.wait_stream(cs)
        self._copy_in(0)
        for i in range(n_steps):
            b = i % 2
            if i + 1 < n_steps:
                self._copy_in((i + 1) % 2)        # overlaps this step's kernels
            cs.wait_event(self.ev_in[b])
            if self.used[b]:
                cs.wait_event(self.ev_out[b])     # the previous result of this set is home
            self.hp.use(self.sets[b])
            self.hp.run_step_kernels(step)
            self.ev_used[b].record(cs)
            self.used[b] = True
            self.d2h.wait_event(self.ev_used[b])
            with torch.cuda.stream(self.d2h):
                self.host_out.copy_(self.sets[b]["out"], non_blocking=True)
            self.ev_out[b].record(self.d2h)
        if end is not None:
            cs.wait_stream(self.d2h)
            cs.wait_stream(self.h2d)
            end.record(cs)
