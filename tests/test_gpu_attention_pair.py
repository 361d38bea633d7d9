"""The CTA-pair form of the active attention (clusters of two CTAs issuing
M = 256 pair MMAs, each CTA staging half of every K/V tile), built with
JANO_ATTN_PAIR=1, against the fp64 oracle through the C ABI.

The product build takes the single-CTA kernel (the pair form measured slower
on B200); this build keeps the pair form correct.  Same tolerances as the
other attention tests: max-abs 2e-2 and mean-rel 5e-3 of the fp64 values.
"""
import ctypes as C
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from workloads import attention_errors, cta_position_rows, oracle_attention_rows

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pair_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    path = build.build(out=os.path.join(ROOT, "_build", "var", "pair", "libjano.so"),
                       defines=("JANO_ATTN_PAIR=1",))
    L = C.CDLL(path)
    P, i, f = C.c_void_p, C.c_int, C.c_float
    L.jano_active_attention.argtypes = [P, P, P, P, i, i, i, i, f, P, P]
    L.jano_get_device_error.argtypes = [P]
    for fn in ("jano_active_attention", "jano_get_device_error"):
        getattr(L, fn).restype = C.c_int
    return L


def _p(t):
    return C.c_void_p(t.data_ptr())


def _run(L, q, k, v, idx):
    N, H, d = k.shape
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ix = torch.from_numpy(idx).cuda()
    assert L.jano_active_attention(_p(qd), _p(kd), _p(vd), _p(ix), idx.size, N, H, d, d ** -0.5,
                                   _p(out), st) == 0
    assert L.jano_get_device_error(st) == 0
    return out.cpu()


@pytest.mark.parametrize("N,n_act,H", [(1, 1, 1),          # one key, one query
                                       (129, 129, 1),      # every token, ragged key tile
                                       (1000, 300, 3),     # the odd CTA of the last pair idle
                                       (2049, 513, 2),     # the last key tile holds one key
                                       (4100, 2000, 2)])   # several pairs, a few key tiles
def test_pair_matches_oracle(pair_lib, N, n_act, H):
    d = 128
    g = np.random.default_rng(N + n_act)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.normal_bf16((n_act, H, d), N + 1)
    k = synth.normal_bf16((N, H, d), N + 2)
    v = synth.normal_bf16((N, H, d), N + 3)
    out = _run(pair_lib, q, k, v, idx)
    rows = np.arange(n_act, dtype=np.int32) if n_act <= 600 else cta_position_rows(n_act, seed=1)
    ref = oracle_attention_rows(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v), rows)
    got = out[torch.from_numpy(idx[rows]).long()].float().numpy()
    mx, mr = attention_errors(got, ref)
    assert mx <= 2e-2 and mr <= 5e-3, (mx, mr)
    mask = torch.ones(N, dtype=torch.bool)
    mask[torch.from_numpy(idx).long()] = False
    assert torch.count_nonzero(out[mask].float()) == 0


def test_pair_equals_single_cta_kernel(pair_lib):
    # the same arithmetic in the same order per row: identical bits
    import kv_cache_analyzer_b200 as J
    from kv_cache_analyzer_b200 import build
    build.build()
    N, n_act, H, d = 3000, 1100, 2, 128
    g = np.random.default_rng(7)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.normal_bf16((n_act, H, d), 71)
    k = synth.normal_bf16((N, H, d), 72)
    v = synth.normal_bf16((N, H, d), 73)
    a = _run(pair_lib, q, k, v, idx)
    b = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(), b, split=1)
    assert J.device_error() == 0
    assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))
