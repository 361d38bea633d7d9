"""GPU parity of the projections of the active rows (gathered linear layer,
scattered output, fused Q/K/V projection with the KV-cache write) against
the fp64 CPU oracle, through the C ABI.

Tolerance, from the arithmetic: BF16 inputs, fp32 accumulation on the tensor
cores, BF16 output rounded to nearest even.  The output rounding contributes
at most 2^-8 |ref| (BF16 unit roundoff is 2^-8 for round-to-nearest with 8
significand bits), and fp32 accumulation of k products at most about
k * 2^-24 * sum_c |x_c w_c| in the worst case; the test allows
2^-8 |ref| + 2^-16 sum_c |x_c w_c| per element, which covers the
accumulation bound up to k = 256 and its square-root growth far beyond,
and checks that the mean relative error sum|gpu - ref| / sum|ref| stays
below 2^-8.  Placement (which rows are written, and that every other row
keeps its bits) is checked bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from workloads import cta_position_rows, oracle_gemm_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


def no_device_error(J):
    code = J.device_error()
    assert code == 0, J.jano_status_str(code)


def f32(bits):
    return synth.bf16_to_f32(bits).astype(np.float64)


def check_rows(got_bits, x_bits, w_bits, src_rows, label=""):
    """got_bits [r][n] BF16 bits of the GPU rows; src_rows the x rows they read."""
    ref = oracle_gemm_rows(x_bits, w_bits, np.asarray(src_rows, dtype=np.int32))
    absdot = np.abs(f32(x_bits)[src_rows]) @ np.abs(f32(w_bits)).T
    got = f32(got_bits)
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * absdot
    worst = np.max(err - bound)
    mean_rel = err.sum() / max(np.abs(ref).sum(), 1e-30)
    print(f"{label}: rows {got.shape[0]}, max-abs {err.max():.3e}, mean-rel {mean_rel:.3e}")
    assert worst <= 0.0, f"{label}: error exceeds bound by {worst:.3e}"
    assert mean_rel <= 2.0 ** -8


@pytest.mark.parametrize("n_x,m,n,k", [(300, 173, 200, 136),    # ragged m, n, k
                                       (130, 129, 256, 64),     # one K block, two row tiles
                                       (1, 1, 8, 8),            # smallest
                                       (1000, 640, 512, 1024)])  # several tiles each way
def test_gather_gemm_matches_oracle(J, n_x, m, n, k):
    gen = np.random.default_rng(n_x + m + n + k)
    x = synth.normal_bf16((n_x, k), seed=n_x + k)
    w = synth.linear_weight_bf16(n, k, seed=n + 7)
    gather = gen.integers(0, n_x, size=m).astype(np.int32)       # repeats allowed
    out = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    J.gather_gemm(x.cuda(), w.cuda(), out, gather=torch.from_numpy(gather).cuda())
    no_device_error(J)
    check_rows(synth.bits_of(out.cpu()), synth.bits_of(x), synth.bits_of(w), gather, f"gather m={m}")


def test_gemm_without_gather_reads_rows_in_order(J):
    x = synth.normal_bf16((200, 96), seed=5)
    w = synth.linear_weight_bf16(136, 96, seed=6)
    out = torch.zeros((200, 136), dtype=torch.bfloat16, device="cuda")
    J.gather_gemm(x.cuda(), w.cuda(), out)
    no_device_error(J)
    check_rows(synth.bits_of(out.cpu()), synth.bits_of(x), synth.bits_of(w), np.arange(200), "plain")


def test_scatter_places_rows_and_keeps_the_rest(J):
    gen = np.random.default_rng(11)
    m, n, k, n_out = 150, 264, 128, 700
    o = synth.normal_bf16((m, k), seed=12)                        # e.g. attention outputs of active rows
    w = synth.linear_weight_bf16(n, k, seed=13)
    dst = np.sort(gen.choice(n_out, size=m, replace=False)).astype(np.int32)
    before = synth.normal_bf16((n_out, n), seed=14)
    y = before.clone().cuda()
    J.gather_gemm(o.cuda(), w.cuda(), y, scatter=torch.from_numpy(dst).cuda())
    no_device_error(J)
    yb, bb = synth.bits_of(y.cpu()), synth.bits_of(before)
    untouched = np.setdiff1d(np.arange(n_out), dst)
    np.testing.assert_array_equal(yb[untouched], bb[untouched])
    check_rows(yb[dst], synth.bits_of(o), synth.bits_of(w), np.arange(m), "scatter")


@pytest.mark.parametrize("N,n_act,heads,d,k", [(1000, 301, 2, 128, 320),   # 256-column tiles
                                               (777, 129, 3, 128, 200),    # hd = 384: 128-column tiles
                                               (64, 64, 1, 128, 64)])      # every token active
def test_qkv_project_matches_oracle_and_writes_only_active_cache_rows(J, N, n_act, heads, d, k):
    gen = np.random.default_rng(N + n_act)
    hd = heads * d
    x = synth.normal_bf16((N, k), seed=N)
    w = synth.linear_weight_bf16(3 * hd, k, seed=k)
    idx = np.sort(gen.choice(N, size=n_act, replace=False)).astype(np.int32)
    kc0, vc0 = synth.normal_bf16((N, hd), seed=1), synth.normal_bf16((N, hd), seed=2)
    q = torch.zeros((n_act, hd), dtype=torch.bfloat16, device="cuda")
    kc, vc = kc0.clone().cuda(), vc0.clone().cuda()
    J.qkv_project(x.cuda(), torch.from_numpy(idx).cuda(), w.cuda(), q, kc, vc)
    no_device_error(J)
    xb, wb = synth.bits_of(x), synth.bits_of(w)
    kb, vb = synth.bits_of(kc.cpu()), synth.bits_of(vc.cpu())
    frozen = np.setdiff1d(np.arange(N), idx)
    np.testing.assert_array_equal(kb[frozen], synth.bits_of(kc0)[frozen])
    np.testing.assert_array_equal(vb[frozen], synth.bits_of(vc0)[frozen])
    check_rows(synth.bits_of(q.cpu()), xb, wb[:hd], idx, "q")
    check_rows(kb[idx], xb, wb[hd:2 * hd], idx, "k")
    check_rows(vb[idx], xb, wb[2 * hd:], idx, "v")


def test_qkv_project_equals_gather_gemm_then_kv_scatter(J):
    # the fused path is the same arithmetic as projecting then scattering: bit for bit
    gen = np.random.default_rng(3)
    N, n_act, heads, d, k = 900, 250, 2, 128, 256
    hd = heads * d
    x = synth.normal_bf16((N, k), seed=21).cuda()
    w = synth.linear_weight_bf16(3 * hd, k, seed=22).cuda()
    idx = torch.from_numpy(np.sort(gen.choice(N, size=n_act, replace=False)).astype(np.int32)).cuda()
    q1 = torch.zeros((n_act, hd), dtype=torch.bfloat16, device="cuda")
    kc1 = torch.zeros((N, heads, d), dtype=torch.bfloat16, device="cuda")
    vc1 = torch.zeros_like(kc1)
    J.qkv_project(x, idx, w, q1, kc1, vc1)
    y = torch.zeros((n_act, 3 * hd), dtype=torch.bfloat16, device="cuda")
    J.gather_gemm(x, w, y, gather=idx)
    kc2, vc2 = torch.zeros_like(kc1), torch.zeros_like(kc1)
    J.kv_scatter(y[:, hd:2 * hd].contiguous().view(n_act, heads, d),
                 y[:, 2 * hd:].contiguous().view(n_act, heads, d), idx, kc2, vc2)
    no_device_error(J)
    assert torch.equal(q1.view(torch.int16), y[:, :hd].contiguous().view(torch.int16))
    assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))


def test_qkv_project_large_video_sampled_rows(J):
    # the large video workload's shapes: 75,600 tokens, hidden 5120 = 40 heads x 128,
    # the 18,900 Active tokens; rows compared (every output column of each):
    # one in each 128-row half and 32-row TMEM lane quarter of 32 spread
    # 256-row tiles, first, last (ragged last tile) and seeded random ones
    N, heads, d = 75600, 40, 128
    hd = k = heads * d
    gen = np.random.default_rng(4)
    idx = np.sort(gen.choice(N, size=N // 4, replace=False)).astype(np.int32)   # 25% Active
    n_act = idx.shape[0]
    x = synth.normal_bf16((N, k), seed=41)
    w = synth.linear_weight_bf16(3 * hd, k, seed=42)
    q = torch.empty((n_act, hd), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((N, hd), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((N, hd), dtype=torch.bfloat16, device="cuda")
    J.qkv_project(x.cuda(), torch.from_numpy(idx).cuda(), w.cuda(), q, kc, vc)
    no_device_error(J)
    rows = np.unique(np.concatenate([cta_position_rows(n_act, n_ctas=32, seed=5),
                                     gen.choice(n_act, size=16, replace=False)]))
    assert rows.size >= 256
    xb, wb = synth.bits_of(x), synth.bits_of(w)
    src = idx[rows]
    check_rows(synth.bits_of(q.cpu())[rows], xb, wb[:hd], src, "large q")
    check_rows(synth.bits_of(kc.cpu())[src], xb, wb[hd:2 * hd], src, "large k")
    check_rows(synth.bits_of(vc.cpu())[src], xb, wb[2 * hd:], src, "large v")


def test_bad_indices_raise_eindex(J):
    x = synth.normal_bf16((64, 64), seed=1).cuda()
    w = synth.linear_weight_bf16(64, 64, seed=2).cuda()
    out = torch.full((8, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    g = torch.tensor([0, 1, 2, 3, 4, 5, 6, 64], dtype=torch.int32, device="cuda")
    J.gather_gemm(x, w, out, gather=g)
    assert J.device_error() == 6                                  # JANO_EINDEX
    assert torch.all(out[7] == 0)                                 # a bad source reads zeros
    out2 = torch.full((8, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    s = torch.tensor([0, 1, 2, 3, 4, 5, 6, 8], dtype=torch.int32, device="cuda")
    J.gather_gemm(x[:8].contiguous(), w, out2, scatter=s)
    assert J.device_error() == 6
    no_device_error(J)                                            # the error word was cleared


def test_qkv_project_rejects_duplicate_and_descending_ids(J):
    # K/V rows go to cache rows idx[i]: ids must be strictly ascending; rows 2
    # (duplicate) and 4 (step back) raise JANO_EINDEX and write no K/V row
    N, hd, k = 16, 128, 64
    idx = np.array([0, 2, 2, 5, 4, 9, 11, 13], dtype=np.int32)
    good = [0, 1, 3, 5, 6, 7]
    x = synth.normal_bf16((N, k), seed=51)
    w = synth.linear_weight_bf16(3 * hd, k, seed=52)
    q = torch.zeros((idx.size, hd), dtype=torch.bfloat16, device="cuda")
    kc0 = synth.normal_bf16((N, hd), seed=53)
    kc, vc = kc0.clone().cuda(), kc0.clone().cuda()
    J.qkv_project(x.cuda(), torch.from_numpy(idx).cuda(), w.cuda(), q, kc, vc)
    assert J.device_error() == 6
    xb, wb = synth.bits_of(x), synth.bits_of(w)
    kb = synth.bits_of(kc.cpu())
    check_rows(kb[idx[good]], xb, wb[hd:2 * hd], idx[good], "k of the valid rows")
    # token 4 is named only by the skipped row: unchanged
    np.testing.assert_array_equal(kb[4], synth.bits_of(kc0)[4])
