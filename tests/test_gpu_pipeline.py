"""The end-to-end step from pinned host memory (``HostStepper``): inputs
copied in and results copied out on their own streams, overlapping the
kernels of the neighbouring steps, with two device sets of buffers.  Its
host result must equal, bit for bit, the result of the same step run on
device-resident inputs, after every step of a pipelined run, and the KV
cache it leaves must be the same too."""
import sys
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _hotpath(J, w, inp, k_cache, v_cache, n_cap, stream):
    from kv_cache_analyzer_b200.pipeline import HotPath
    hp = HotPath(K=w.K, C=w.C, latent_geom=J.Geometry(w.F, w.H, w.W, w.block, w.patch),
                 token_geom=J.Geometry(w.F, w.H, w.W, w.patch, w.patch), heads=w.heads, d=w.d,
                 frac_active=w.frac_active, frac_static=w.frac_static,
                 sched=J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static),
                 device="cuda", stream=stream)
    hp.set_activations(n_cap)
    with torch.cuda.stream(stream):
        hp.lat.copy_(inp["lat"]); hp.field.copy_(inp["field"])
        hp.q_act.copy_(inp["q_act"]); hp.k_act.copy_(inp["k_act"]); hp.v_act.copy_(inp["v_act"])
        hp.k_cache.copy_(k_cache); hp.v_cache.copy_(v_cache)
    stream.synchronize()
    hp.plan()
    return hp


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_pipelined_host_steps_equal_device_steps(name):
    import bench
    import synth
    import kv_cache_analyzer_b200 as J
    from kv_cache_analyzer_b200.pipeline import HostStepper
    w = synth.WORKLOADS[name]
    inp, k_cache, v_cache, n_cap = bench.make_inputs(w)
    stream = torch.cuda.Stream()
    # device-resident reference
    ref = _hotpath(J, w, inp, k_cache, v_cache, n_cap, stream)
    step = w.warmup
    _, n_act = ref.due(step)
    ref.run_step_kernels(step)
    stream.synchronize()
    assert J.device_error() == 0
    out_ref = ref.out.cpu()
    kc_ref = ref.k_cache.cpu()
    # pipelined from pinned host memory, three steps
    hp = _hotpath(J, w, inp, k_cache, v_cache, n_cap, stream)
    host = {k: v.pin_memory() for k, v in inp.items()}
    for k in ("q_act", "k_act", "v_act"):
        host[k] = host[k][:n_act]
    host_out = torch.full(hp.out.shape, 7.0, dtype=hp.out.dtype).pin_memory()
    st = HostStepper(hp, host, host_out)
    st.run(step, 3)
    torch.cuda.synchronize()
    assert J.device_error() == 0
    assert torch.equal(host_out.view(torch.int16), out_ref.view(torch.int16))
    assert torch.equal(hp.k_cache.cpu().view(torch.int16), kc_ref.view(torch.int16))


def test_whole_step_is_deterministic_over_10_reruns():
    # fixed reduction orders everywhere: scores, levels, schedule, the
    # scattered cache and the attention output repeat bit for bit
    import bench
    import synth
    import kv_cache_analyzer_b200 as J
    w = synth.WORKLOADS["small"]
    inp, k_cache, v_cache, n_cap = bench.make_inputs(w)
    stream = torch.cuda.Stream()
    hp = _hotpath(J, w, inp, k_cache, v_cache, n_cap, stream)
    step = w.warmup
    first = None
    for _ in range(10):
        hp.k_cache.copy_(k_cache.cuda()); hp.v_cache.copy_(v_cache.cuda()); hp.out.zero_()
        torch.cuda.synchronize()
        hp.run_step_kernels(step)
        stream.synchronize()
        snap = [t.clone() for t in (hp.scores, hp.levels, hp.offsets, hp.idx, hp.k_cache, hp.out)]
        if first is None:
            first = snap
        else:
            for a, b in zip(first, snap):
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert J.device_error() == 0
