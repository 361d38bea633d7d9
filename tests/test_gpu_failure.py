"""Failure detection on the GPU, without a fault: a bounded wait runs out.

A test-only build of the library (``-DJANO_INJECT_DROP_LOAD=2``) leaves one
copy unissued in the attention and projection producers, so the MMA
thread's wait for that stage can never complete.  Every wait in those
kernels is bounded (about a second); the CTA records JANO_ETIMEOUT on the
device error word, the other warps see its abort flag, copies already in
flight are drained, tensor memory is freed and the kernel returns.  The
host reads the status; the context stays usable, which the product library
then shows by computing the same attention correctly.  Nothing here traps,
faults or hangs the GPU.
"""
import ctypes as C
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ETIMEOUT = 7


@pytest.fixture(scope="module")
def inject_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    path = build.build(out=os.path.join(ROOT, "_build", "inject", "libjano_inject.so"),
                       defines=("JANO_INJECT_DROP_LOAD=2",))
    L = C.CDLL(path)
    P, i, f = C.c_void_p, C.c_int, C.c_float
    L.jano_active_attention.argtypes = [P, P, P, P, i, i, i, i, f, P, P]
    L.jano_qkv_project.argtypes = [P, i, P, i, P, i, i, P, P, P, P]
    L.jano_active_attention_split.argtypes = [P, P, P, P, i, i, i, i, f, i, P, C.c_size_t, P, P]
    L.jano_active_attention_workspace_bytes.argtypes = [i, i, i, i]
    L.jano_active_attention_workspace_bytes.restype = C.c_size_t
    L.jano_get_device_error.argtypes = [P]
    for fn in ("jano_active_attention", "jano_active_attention_split", "jano_qkv_project",
               "jano_get_device_error"):
        getattr(L, fn).restype = C.c_int
    return L


def _p(t):
    return C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _attention_case():
    gen = np.random.default_rng(1)
    N, n_act, H, d = 512, 128, 1, 128
    q = synth.normal_bf16((n_act, H, d), 1)
    kc = synth.normal_bf16((N, H, d), 2)
    vc = synth.normal_bf16((N, H, d), 3)
    idx = np.sort(gen.choice(N, size=n_act, replace=False)).astype(np.int32)
    return q, kc, vc, idx


def test_attention_wait_runs_out_and_reports_etimeout(inject_lib):
    L = inject_lib
    q, kc, vc, idx = _attention_case()
    N, H, d = kc.shape
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    ix = torch.from_numpy(idx).cuda()
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    assert L.jano_active_attention(_p(qd), _p(kd), _p(vd), _p(ix), idx.size, N, H, d, d ** -0.5,
                                   _p(out), _stream()) == 0
    code = L.jano_get_device_error(_stream())         # synchronises
    wall = time.perf_counter() - t0
    assert code == ETIMEOUT, code
    assert wall < 30.0, wall
    assert L.jano_get_device_error(_stream()) == 0    # read and cleared


def test_split_attention_timeout_leaves_rows_untouched(inject_lib):
    # 384 keys = 3 key tiles in 2 ranges: range 0 takes tile 0 (two loads, none
    # dropped) and completes; range 1 takes tiles 1-2, its third load is never
    # issued and it times out.  The merge must then skip every row (one of its
    # partials is missing) instead of reading the range's unwritten workspace,
    # so `out` keeps its contents, as with the unsplit kernel.
    L = inject_lib
    gen = np.random.default_rng(2)
    N, n_act, H, d, n_split = 384, 128, 1, 128, 2
    q = synth.normal_bf16((n_act, H, d), 11).cuda()
    kc = synth.normal_bf16((N, H, d), 12).cuda()
    vc = synth.normal_bf16((N, H, d), 13).cuda()
    ix = torch.from_numpy(np.sort(gen.choice(N, size=n_act, replace=False)).astype(np.int32)).cuda()
    out = torch.full((N, H, d), 0.25, dtype=torch.bfloat16, device="cuda")
    nb = L.jano_active_attention_workspace_bytes(n_act, H, d, n_split)
    # garbage in the workspace, as a reused buffer would hold
    ws = torch.full((nb // 4,), float("nan"), dtype=torch.float32, device="cuda")
    assert L.jano_active_attention_split(_p(q), _p(kc), _p(vc), _p(ix), n_act, N, H, d, d ** -0.5,
                                         n_split, _p(ws), nb, _p(out), _stream()) == 0
    assert L.jano_get_device_error(_stream()) == ETIMEOUT
    assert L.jano_get_device_error(_stream()) == 0
    assert torch.all(out == 0.25)


def test_projection_wait_runs_out_and_reports_etimeout(inject_lib):
    L = inject_lib
    N, n_act, hd, k = 300, 256, 128, 512
    x = synth.normal_bf16((N, k), 4).cuda()
    w = synth.linear_weight_bf16(3 * hd, k, 5).cuda()
    idx = torch.arange(0, 2 * n_act, 2, dtype=torch.int32, device="cuda") % N
    idx = torch.unique(idx).to(torch.int32)
    q = torch.zeros(idx.numel(), hd, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(N, hd, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    assert L.jano_qkv_project(_p(x), N, _p(idx), idx.numel(), _p(w), hd, k, _p(q), _p(kc), _p(vc),
                              _stream()) == 0
    assert L.jano_get_device_error(_stream()) == ETIMEOUT
    assert L.jano_get_device_error(_stream()) == 0


def test_context_still_computes_after_the_timeouts(inject_lib):
    # the product library on the same device, after the timed-out launches
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as J
    q, kc, vc, idx = _attention_case()
    N, H, d = kc.shape
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(idx).cuda(), out)
    assert J.device_error() == 0
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(kc), synth.bits_of(vc))
    got = out.cpu()[torch.from_numpy(idx).long()].float().numpy()
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 and err.sum() / np.abs(ref).sum() <= 5e-3
