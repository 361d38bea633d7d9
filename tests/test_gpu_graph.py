"""The step captured as a CUDA graph (HotPath.capture_step) and replayed:
every output -- block scores, levels, schedule, the KV cache after the
scatter, the attention rows -- bit for bit equal to the same step run
launch by launch; and graphs of back-to-back classify / schedule launches
(HotPath.capture_repeated) leave the same results as one launch."""
import os
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else
                               (torch.uint8 if t.dtype == torch.uint8 else torch.int32)).cpu()


def _hot_path(J, w, stream):
    import bench
    from kv_cache_analyzer_b200.pipeline import HotPath
    inp, k_cache, v_cache, n_cap = bench.make_inputs(w)
    hp = HotPath(K=w.K, C=w.C, latent_geom=J.Geometry(w.F, w.H, w.W, w.block, w.patch),
                 token_geom=J.Geometry(w.F, w.H, w.W, w.patch, w.patch), heads=w.heads, d=w.d,
                 frac_active=w.frac_active, frac_static=w.frac_static,
                 sched=J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static),
                 stream=stream)
    hp.set_activations(n_cap)
    with torch.cuda.stream(stream):
        hp.lat.copy_(inp["lat"]); hp.field.copy_(inp["field"])
        hp.q_act.copy_(inp["q_act"]); hp.k_act.copy_(inp["k_act"]); hp.v_act.copy_(inp["v_act"])
        hp.k_cache.copy_(k_cache); hp.v_cache.copy_(v_cache)
    stream.synchronize()
    hp.plan()
    return hp, k_cache, v_cache


def _outputs(hp):
    n_idx = int(hp.offsets[-1].item())          # the schedule's entries; the rest is unused
    return {"scores": _bits(hp.scores), "levels": _bits(hp.levels), "offsets": _bits(hp.offsets),
            "idx": _bits(hp.idx[:n_idx]), "k_cache": _bits(hp.k_cache), "v_cache": _bits(hp.v_cache),
            "out": _bits(hp.out)}


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_step_graph_equals_eager_step(name):
    import synth
    import kv_cache_analyzer_b200 as J
    w = synth.WORKLOADS[name]
    stream = torch.cuda.Stream()
    hp, k0, v0 = _hot_path(J, w, stream)
    step = w.warmup
    # eager step from the initial cache
    hp.run_step_kernels(step)
    stream.synchronize()
    assert J.device_error(stream) == 0
    eager = _outputs(hp)
    # graph: capture (after one ordinary pass), restore the inputs the step
    # changes (cache, out), replay once
    g = hp.capture_step(step)
    with torch.cuda.stream(stream):
        hp.k_cache.copy_(k0); hp.v_cache.copy_(v0); hp.out.zero_()
        hp.scores.zero_(); hp.levels.zero_(); hp.idx.zero_()
        g.replay()
    stream.synchronize()
    assert J.device_error(stream) == 0
    got = _outputs(hp)
    for k in eager:
        assert torch.equal(eager[k], got[k]), k
    del g


def test_repeated_plan_kernels_in_a_graph():
    import synth
    import kv_cache_analyzer_b200 as J
    w = synth.WORKLOADS["small"]
    stream = torch.cuda.Stream()
    hp, _, _ = _hot_path(J, w, stream)
    n_idx = int(hp.offsets[-1].item())
    ref_levels, ref_off, ref_idx = _bits(hp.levels), _bits(hp.offsets), _bits(hp.idx[:n_idx])
    cls = hp.capture_repeated(
        lambda s: J.jano_classify(hp.field, hp.field.numel(), hp.frac_active, hp.frac_static, hp.levels, s), 5)
    sch = hp.capture_repeated(
        lambda s: J.jano_build_schedule(hp.levels, hp._tgc, hp._sc, hp.offsets, hp.idx, hp.idx.numel(),
                                        hp.token_levels, hp.ws, hp.ws_bytes, s), 5)
    with torch.cuda.stream(stream):
        hp.levels.zero_(); hp.offsets.zero_(); hp.idx.zero_()
        cls.replay()
        sch.replay()
    stream.synchronize()
    assert J.device_error(stream) == 0
    assert torch.equal(_bits(hp.levels), ref_levels)
    assert torch.equal(_bits(hp.offsets), ref_off)
    assert torch.equal(_bits(hp.idx[:n_idx]), ref_idx)
    del cls, sch
