"""GPU parity of the method variants next to the hot path: the random-masking
ablation's scores and level maps (bit-exact: counter-based generator and
integer ranks), the Static refresh period of the pages' example (every
5th step), the literal score reading and the FFT baseline score, through the
C ABI."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


@pytest.mark.parametrize("n,seed", [(1, 0), (1000, 7), (8190, 2**63 + 5), (19320, 123456789)])
def test_random_scores_bit_exact(J, n, seed):
    got = J.random_scores(n, seed).cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), oracle.random_scores(n, seed).view(np.uint32))


@pytest.mark.parametrize("n,fa,fs", [(19320, 0.25, 0.45), (4096, 0.30, 0.40), (257, 0.35, 0.65)])
def test_random_level_map_bit_exact_with_jano_counts(J, n, fa, fs):
    lv = J.classify(J.random_scores(n, 42), fa, fs).cpu().numpy()
    assert J.device_error() == 0
    ref = oracle.classify(oracle.random_scores(n, 42), fa, fs)
    np.testing.assert_array_equal(lv, ref)
    n_a, n_s = oracle.level_counts(n, fa, fs)
    assert (lv == 3).sum() == n_a and (lv == 1).sum() == n_s
    # a different seed moves the levels, not their counts
    lv2 = J.classify(J.random_scores(n, 43), fa, fs).cpu().numpy()
    assert (lv2 == 3).sum() == n_a and not np.array_equal(lv, lv2)


def test_schedule_static_every_5th_step_bit_exact(J):
    g = np.random.default_rng(9)
    F, H, W = 3, 12, 14
    lv = g.integers(1, 4, size=F * 6 * 7).astype(np.uint8)
    sched = J.Schedule(50, 5, 5, 2, 5)
    geom = J.Geometry(F, H, W, (1, 2, 2), (1, 2, 2))
    off, idx, tl = J.build_schedule(torch.from_numpy(lv).cuda(), geom, sched)
    assert J.device_error() == 0
    roff, ridx, rtl = oracle.build_schedule(lv, (F, H, W), (1, 2, 2), (1, 2, 2), 50, 5, 5, 2, 5)
    np.testing.assert_array_equal(off.cpu().numpy(), roff)
    np.testing.assert_array_equal(idx.cpu().numpy()[: roff[-1]], ridx)
    np.testing.assert_array_equal(tl.cpu().numpy(), rtl)


# ---------------------------------------------------------------- literal score reading
@pytest.mark.parametrize("name", ["tiny", "image", "small", "large"])
def test_literal_scores_match_oracle(J, name):
    """fp32 on the GPU, fp64 in the oracle.  The literal score takes
    differences of second differences, whose fp32 rounding is absolute (a few
    units of 2^-24 max|x|) while the scores of smooth content are small, so
    the bound is 1e-5 |ref| + 2^-19 max|x| per block."""
    import synth
    from workloads import latent
    w = synth.WORKLOADS[name]
    lat = latent(name)
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    got = J.block_scores_literal(torch.from_numpy(lat).cuda(), geom).cpu().numpy()
    assert J.device_error() == 0
    ref = oracle.block_scores_literal(lat, w.block)
    bound = 1e-5 * np.abs(ref) + 2.0 ** -19 * float(np.abs(lat).max())
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))
    again = J.block_scores_literal(torch.from_numpy(lat).cuda(), geom).cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), again.view(np.uint32))


@pytest.mark.parametrize("shape,block", [((3, 2, 3, 9, 12), (1, 4, 4)), ((4, 3, 5, 6, 8), (2, 3, 2)),
                                         ((6, 1, 1, 16, 16), (1, 2, 2)), ((3, 1, 2, 4, 20), (1, 4, 8))])
def test_literal_scores_edge_geometries(J, shape, block):
    g = np.random.default_rng(sum(shape) + 1)
    lat = g.standard_normal(shape).astype(np.float32)
    K1, Cc, F, H, W = shape
    got = J.block_scores_literal(torch.from_numpy(lat).cuda(), J.Geometry(F, H, W, block, (1, 1, 1))).cpu().numpy()
    ref = oracle.block_scores_literal(lat, block)
    bound = 1e-5 * np.abs(ref) + 2.0 ** -19 * float(np.abs(lat).max())
    assert np.all(np.abs(got - ref) <= bound)


# ---------------------------------------------------------------- FFT baseline score
def _fft_bound(x, block, ref):
    """fp32 against fp64, from the arithmetic: each DFT bin is a sum of n_b
    terms (twiddles exact or correctly rounded), so its error is at most
    about (n_b + 2) 2^-24 sum|x|; squared, summed over at most n_b bins and
    divided by n_b^2 that is 2 (n_b + 2) 2^-24 n_b M_b with M_b the channel
    mean of (mean |x| over the block)^2.  Bound: 2^-16 |ref| + that."""
    Cc, F, H, W = x.shape
    bf, bh, bw = block
    ax = np.abs(x.astype(np.float64))
    out = np.empty_like(ref)
    b = 0
    for f0 in range(0, F, bf):
        for h0 in range(0, H, bh):
            for w0 in range(0, W, bw):
                blk = ax[:, f0:f0 + bf, h0:h0 + bh, w0:w0 + bw]
                n = blk[0].size
                M = np.mean(blk.reshape(Cc, -1).mean(axis=1) ** 2)
                out[b] = 2.0 ** -16 * abs(ref[b]) + 2 * (n + 2) * 2.0 ** -24 * n * M
                b += 1
    return out


@pytest.mark.parametrize("name", ["tiny", "image", "small", "large"])
@pytest.mark.parametrize("cutoff", [1, 2])
def test_fft_scores_match_oracle(J, name, cutoff):
    import synth
    from workloads import latent
    w = synth.WORKLOADS[name]
    x = np.ascontiguousarray(latent(name)[w.K])          # the last warm-up snapshot
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    xd = torch.from_numpy(x).cuda()
    got = J.fft_scores(xd, geom, cutoff).cpu().numpy()
    assert J.device_error() == 0
    ref = oracle.fft_scores(x, w.block, cutoff)
    err = np.abs(got - ref) - _fft_bound(x, w.block, ref)
    assert np.all(err <= 0), float(err.max())
    again = J.fft_scores(xd, geom, cutoff).cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), again.view(np.uint32))


@pytest.mark.parametrize("shape,block", [((2, 3, 9, 12), (1, 4, 4)), ((3, 5, 6, 8), (2, 3, 2)),
                                         ((1, 1, 16, 16), (1, 2, 2)), ((1, 2, 4, 20), (1, 4, 8)),
                                         ((4, 3, 19, 21), (1, 8, 8)), ((3, 5, 7, 9), (2, 2, 2)),
                                         ((2, 5, 10, 13), (2, 4, 4)), ((1, 7, 9, 11), (4, 4, 4)),
                                         ((2, 3, 7, 11), (1, 4, 4)), ((9, 3, 10, 12), (1, 4, 4)),
                                         ((6, 2, 9, 10), (2, 4, 4)), ((11, 2, 16, 24), (1, 8, 8))])
@pytest.mark.parametrize("cutoff", [0, 1, 2, 3])
def test_fft_scores_edge_geometries(J, shape, block, cutoff):
    # partial blocks on every axis (FFT lengths below the block's, and edge
    # lengths 3, 5, 7 that take the direct DFT), each specialised block shape
    # and the generic one, channel counts below and above the channel groups
    # (the prefetching walk), unaligned rows (W not a multiple of 4), and
    # cutoffs from "all bins" (the mean square) to above every folded index
    # (exactly 0)
    g = np.random.default_rng(sum(shape) + cutoff)
    x = (g.standard_normal(shape) * 2.0 + 0.5).astype(np.float32)
    Cc, F, H, W = shape
    got = J.fft_scores(torch.from_numpy(x).cuda(), J.Geometry(F, H, W, block, (1, 1, 1)), cutoff)
    got = got.cpu().numpy()
    assert J.device_error() == 0
    ref = oracle.fft_scores(x, block, cutoff)
    assert np.all(np.abs(got - ref) <= _fft_bound(x, block, ref))
    assert np.array_equal(got == 0, ref == 0)            # empty bands give exact zeros


# ---------------------------------------------------------------- read-rate calibration
@pytest.mark.parametrize("n,n_partial", [(4, 1), (1000, 7), (1 << 20, 148), (3_000_004, 148), (64, 148)])
def test_stream_sum_partials(J, n, n_partial):
    # jano_stream_sum (the one-pass read the analyzer's HBM rate is compared
    # with): partial[i] is the fp32 sum of the i-th contiguous share of
    # ceil(n/4 / n_partial) float4s; checked against fp64 sums of the same shares
    g = np.random.default_rng(n)
    x = g.standard_normal(n).astype(np.float32)
    out = J.stream_sum(torch.from_numpy(x).cuda(), n_partial).cpu().numpy()
    assert J.device_error() == 0
    per = -(-(n // 4) // n_partial) * 4
    ref = np.array([x[i * per:(i + 1) * per].astype(np.float64).sum() for i in range(n_partial)])
    mag = np.array([np.abs(x[i * per:(i + 1) * per]).astype(np.float64).sum() for i in range(n_partial)])
    assert np.all(np.abs(out - ref) <= 1e-5 * mag + 1e-6)
