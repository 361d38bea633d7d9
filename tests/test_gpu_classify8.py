"""The portable 8-CTA form of jano_classify (built with
JANO_CLASSIFY_CLUSTER=8; devices that run 16-CTA clusters take the 16-CTA
form) against the fp64 oracle through the C ABI: bit-exact levels on ties,
sizes and the value distributions that exercise every route of the select."""
import ctypes as C
import os

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib8():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    path = build.build(out=os.path.join(ROOT, "_build", "var", "cls8", "libjano.so"),
                       defines=("JANO_CLASSIFY_CLUSTER=8",))
    L = C.CDLL(path)
    P = C.c_void_p
    L.jano_classify.argtypes = [P, C.c_int, C.c_float, C.c_float, P, P]
    L.jano_classify.restype = C.c_int
    L.jano_get_device_error.argtypes = [P]
    L.jano_get_device_error.restype = C.c_int
    return L


def _classify(L, s, fa, fs):
    x = torch.from_numpy(s).cuda()
    lv = torch.empty(s.size, dtype=torch.uint8, device="cuda")
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.jano_classify(C.c_void_p(x.data_ptr()), s.size, fa, fs, C.c_void_p(lv.data_ptr()), st) == 0
    assert L.jano_get_device_error(st) == 0
    return lv.cpu().numpy()


def _scores(kind, n, seed):
    g = np.random.default_rng(seed)
    if kind == "ties":
        return g.choice(np.array([-2.0, -0.0, 0.0, 0.5, 0.5, 1.0, 3.0], dtype=np.float32), size=n)
    if kind == "normal":
        return g.standard_normal(n).astype(np.float32)
    if kind == "outliers":
        s = g.standard_normal(n)
        s[g.choice(n, 3, replace=False)] = [1e30, -1e30, 2e29]
        return s.astype(np.float32)
    return (g.lognormal(0.0, 4.0, n)).astype(np.float32)


@pytest.mark.parametrize("kind,n", [("ties", 1), ("ties", 1025), ("ties", 100_003), ("normal", 75_600),
                                    ("normal", 400_003), ("outliers", 75_600), ("lognormal", 32_760)])
def test_cluster8_matches_oracle(lib8, kind, n):
    s = _scores(kind, n, n)
    for fa, fs in [(0.25, 0.45), (0.3, 0.4), (0.0, 0.5), (1.0, 0.0)]:
        np.testing.assert_array_equal(_classify(lib8, s, fa, fs), oracle.classify(s, fa, fs),
                                      err_msg=f"{kind} {n} {fa},{fs}")
