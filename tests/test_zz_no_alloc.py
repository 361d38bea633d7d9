"""jano_build_schedule_noalloc, the schedule builder for callers that cannot
allocate device memory (plug-ins handed fixed buffers by a host framework,
runtimes without a device allocator, hosts whose pool forbids side
allocations).  It uses the library's own 1 MiB device array as scratch
instead of a caller workspace.

Called through the C ABI, its outputs must equal those of jano_build_schedule
(with a caller workspace) bit for bit, on two calls in a row with different
inputs, so contents left in the shared array by one call cannot leak into
the next.  This file is collected last; it also passes alone in a fresh
process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


def _run_both(J, levels_np, geom, sched):
    L = J.lib()
    dev = torch.device("cuda")
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    g, c = geom.c(), sched.c()
    N = geom.n_tokens
    levels = torch.from_numpy(levels_np).to(dev)
    outs = []
    for variant in ("workspace", "noalloc"):
        off = torch.full((sched.T + 1,), -7, dtype=torch.int32, device=dev)
        idx = torch.full((sched.T * N,), -7, dtype=torch.int32, device=dev)
        tl = torch.full((N,), 0xEE, dtype=torch.uint8, device=dev)
        P = lambda t: C.c_void_p(t.data_ptr())
        if variant == "workspace":
            nb = L.jano_build_schedule_workspace_bytes(C.byref(g))
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
            code = L.jano_build_schedule(P(levels), C.byref(g), C.byref(c), P(off), P(idx),
                                         idx.numel(), P(tl), P(ws), nb, st)
        else:
            code = L.jano_build_schedule_noalloc(P(levels), C.byref(g), C.byref(c), P(off),
                                                 P(idx), idx.numel(), P(tl), st)
        assert code == 0, J.jano_status_str(code)
        torch.cuda.synchronize()
        o = off.cpu().numpy()
        outs.append((o, idx.cpu().numpy()[: o[-1]], tl.cpu().numpy()))
    assert J.device_error() == 0
    (o1, i1, t1), (o2, i2, t2) = outs
    np.testing.assert_array_equal(o2, o1)
    np.testing.assert_array_equal(i2, i1)
    np.testing.assert_array_equal(t2, t1)
    return o1


def test_noalloc_schedule_matches_workspace_variant_on_two_calls(J):
    import synth
    w = synth.WORKLOADS["large"]
    sched = J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static)
    # call 1: the large video geometry, analyzer blocks mapped onto tokens
    g1 = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    lv1 = np.random.default_rng(1).integers(1, 4, size=g1.n_blocks).astype(np.uint8)
    off1 = _run_both(J, lv1, g1, sched)
    # call 2: a smaller geometry with another level map, right after
    g2 = J.Geometry(3, 20, 36, (1, 2, 2), (1, 2, 2))
    lv2 = np.random.default_rng(2).integers(1, 4, size=g2.n_blocks).astype(np.uint8)
    off2 = _run_both(J, lv2, g2, J.Schedule(12, 2, 2, 3, 5))
    assert off1[-1] > off2[-1] > 0


def test_noalloc_at_its_exact_limit_matches_workspace_variant(J):
    # 2699 x 384 = 1,036,416 tokens fill the 1 MiB scratch exactly
    g = J.Geometry(1, 2699, 384, (1, 4, 4), (1, 1, 1))
    assert J.jano_build_schedule_workspace_bytes(g.c()) == 1 << 20
    lv = np.random.default_rng(3).integers(1, 4, size=g.n_blocks).astype(np.uint8)
    off = _run_both(J, lv, g, J.Schedule(3, 1, 1, 1, 1))
    assert off[-1] > 0


def test_noalloc_rejects_geometry_beyond_its_scratch(J):
    L = J.lib()
    big = J.Geometry(1, 1, 1_036_417, (1, 1, 1), (1, 1, 1)).c()   # one token over the limit
    c = J.Schedule(2, 1, 1, 1, 1).c()
    fake = C.c_void_p(256)
    assert L.jano_build_schedule_noalloc(fake, C.byref(big), C.byref(c), fake, fake, 10**9, None,
                                         None) == 4
