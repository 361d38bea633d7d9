"""Pins for the fp64 CPU oracle: it is checked against things other than itself.

Hand-worked examples (tests/golden), closed forms, invariants, library
routines (numpy sorting and indexing, torch's scaled-dot-product attention in
fp64) and brute force on tiny inputs.  Each pin is chosen so that a plausible
mistake in the oracle -- a dropped term, a wrong weight, a wrong neighbour, a
squared instead of absolute difference, an off-by-one step window, a wrong
tie-break, a wrong refresh phase -- fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from conftest import golden


# ---------------------------------------------------------------- o1 scores
def test_block_scores_hand_example():
    g = golden("block_scores_hand.json")
    lat = np.array(g["lat"], dtype=np.float32)
    for case in g["cases"]:
        got = oracle.block_scores(lat, tuple(case["block"]))
        np.testing.assert_allclose(got, case["expected"], rtol=1e-14, atol=1e-14)


def test_block_scores_constant_latent_is_zero():
    lat = np.full((6, 3, 4, 8, 8), 2.75, dtype=np.float32)
    assert np.all(oracle.block_scores(lat, (1, 4, 4)) == 0.0)


def test_block_scores_temporally_affine_is_zero():
    # x_k = a + k b, spatially constant per channel: no second difference, no gradient
    K = 5
    a = np.array([0.5, -1.0, 2.0])
    b = np.array([0.25, 1.5, -0.75])
    lat = np.empty((K + 1, 3, 2, 4, 4), dtype=np.float32)
    for k in range(K + 1):
        lat[k] = (a + k * b)[:, None, None, None]
    assert np.all(oracle.block_scores(lat, (1, 2, 2)) == 0.0)


def test_block_scores_spatial_gradient_closed_form():
    # x = alpha*h + beta*w (constant in k and f): term = 0.5*sqrt(alpha^2+beta^2)
    # where both neighbours exist, 0.5*|alpha| on the last column, 0.5*|beta|
    # on the last row, 0 in the corner.
    K, F, H, W = 3, 1, 8, 8
    alpha, beta = 3.0, 4.0
    hh, ww = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    x = (alpha * hh + beta * ww).astype(np.float32)
    lat = np.broadcast_to(x, (K + 1, 2, F, H, W)).copy()
    s = oracle.block_scores(lat, (1, 4, 4)).reshape(2, 2)
    assert s[0, 0] == pytest.approx(0.5 * 5.0, rel=1e-15)
    # block (0,1) holds the last column: 12 elements with 5, 4 with |alpha|=3
    assert s[0, 1] == pytest.approx(0.5 * (12 * 5.0 + 4 * 3.0) / 16, rel=1e-15)
    # block (1,0) holds the last row: 12 with 5, 4 with |beta|=4
    assert s[1, 0] == pytest.approx(0.5 * (12 * 5.0 + 4 * 4.0) / 16, rel=1e-15)
    # block (1,1): 9 with 5, 3 with 3, 3 with 4, corner 0
    assert s[1, 1] == pytest.approx(0.5 * (9 * 5.0 + 3 * 3.0 + 3 * 4.0) / 16, rel=1e-15)


def test_block_scores_temporal_gradient_closed_form():
    # x = gamma*f: term = 0.5*|gamma| for f < F-1, 0 on the last frame
    K, F, H, W = 2, 3, 4, 4
    gamma = -1.5
    x = (gamma * np.arange(F, dtype=np.float64))[:, None, None] * np.ones((F, H, W))
    lat = np.broadcast_to(x.astype(np.float32), (K + 1, 1, F, H, W)).copy()
    s = oracle.block_scores(lat, (1, 4, 4))
    np.testing.assert_allclose(s, [0.75, 0.75, 0.0], rtol=1e-15)
    s2 = oracle.block_scores(lat, (3, 4, 4))
    assert s2[0] == pytest.approx(0.75 * 2 / 3, rel=1e-15)


def test_block_scores_second_difference_closed_form():
    # x_k = n_c + s_k G_c, spatially constant per channel:
    # S = mean_c |G_c| * mean_{k=1..K-1} |s_{k+1} - 2 s_k + s_{k-1}|
    K = 5
    s = np.array([0.0, 0.3, 0.1, 0.9, 0.4, 1.0])
    G = np.array([1.0, -2.0, 0.5, 3.0])
    n = np.array([0.1, 0.2, -0.3, 0.4])
    lat = np.empty((K + 1, 4, 2, 4, 4), dtype=np.float64)
    for k in range(K + 1):
        lat[k] = (n + s[k] * G)[:, None, None, None]
    lat32 = lat.astype(np.float32)
    # closed form evaluated on the fp32-rounded snapshots (the oracle's input)
    per_c = lat32[:, :, 0, 0, 0].astype(np.float64)
    d2 = np.abs(per_c[2:] - 2 * per_c[1:-1] + per_c[:-2])      # [K-1, C]
    expect = d2.mean()
    got = oracle.block_scores(lat32, (1, 2, 2))
    np.testing.assert_allclose(got, expect, rtol=1e-14)
    # and against the exact-real closed form, within fp32 input rounding
    exact = np.mean(np.abs(G)) * np.mean(np.abs(s[2:] - 2 * s[1:-1] + s[:-2]))
    np.testing.assert_allclose(got, exact, rtol=1e-6)


def test_block_scores_step_window_uses_k1_to_km1():
    # Changing x_0 only touches the k=1 second difference; gradients of x_0
    # must not enter.  A spatial ramp placed in x_0 alone changes the score
    # only through |x_2 - 2x_1 + x_0|.
    K, F, H, W = 3, 1, 4, 4
    lat = np.zeros((K + 1, 1, F, H, W), dtype=np.float32)
    lat[0, 0, 0] = np.arange(H * W, dtype=np.float32).reshape(H, W)
    got = oracle.block_scores(lat, (1, 4, 4))
    expect = np.arange(H * W).mean() / (K - 1)
    assert got[0] == pytest.approx(expect, rel=1e-15)
    # x_K only enters the k=K-1 second difference
    lat2 = np.zeros_like(lat)
    lat2[K, 0, 0] = 2.0
    assert oracle.block_scores(lat2, (1, 4, 4))[0] == pytest.approx(2.0 / (K - 1), rel=1e-15)


def test_block_scores_invariances():
    w = synth.WORKLOADS["tiny"]
    lat = synth.latent_history(w.K, 4, 2, 12, 12, seed=11)
    base = oracle.block_scores(lat, (1, 4, 4))
    # channel permutation
    perm = oracle.block_scores(lat[:, ::-1].copy(), (1, 4, 4))
    np.testing.assert_allclose(perm, base, rtol=1e-13)
    # a constant offset is removed by every difference: x -> x + 1024 is exact
    # in fp32 only up to the inputs' rounding, so compare within that
    shifted = oracle.block_scores(lat + np.float32(1024.0), (1, 4, 4))
    np.testing.assert_allclose(shifted, base, rtol=2e-3)
    # positive homogeneity of degree one (scaling by a power of two is exact)
    np.testing.assert_allclose(oracle.block_scores(lat * np.float32(4.0), (1, 4, 4)), 4.0 * base, rtol=1e-14)
    np.testing.assert_allclose(oracle.block_scores(-lat, (1, 4, 4)), base, rtol=1e-14)


def test_block_scores_partial_edge_blocks():
    # H=6 with bh=4: the second block row holds two rows; each block averages
    # over its real elements only.  A latent with |d2| = 1 everywhere and no
    # gradient scores exactly 1 in every block, full or partial.
    K, F, H, W = 2, 1, 6, 6
    lat = np.zeros((K + 1, 1, F, H, W), dtype=np.float32)
    lat[2] = 1.0
    got = oracle.block_scores(lat, (1, 4, 4))
    np.testing.assert_array_equal(got, np.ones(4))


def test_block_scores_brute_force_tiny():
    # Brute force on a 2x2x2 latent with C=2: the score of the single block is
    # the average of the per-element terms written out from the definition,
    # one python expression per element.
    gen = np.random.default_rng(5)
    lat = gen.standard_normal((4, 2, 2, 2, 2)).astype(np.float32)
    x = lat.astype(np.float64)
    total = 0.0
    for k in (1, 2):
        for c in range(2):
            for f in range(2):
                for h in range(2):
                    for w in range(2):
                        d2 = abs(x[k + 1, c, f, h, w] - 2 * x[k, c, f, h, w] + x[k - 1, c, f, h, w])
                        df = x[k, c, 1, h, w] - x[k, c, 0, h, w] if f == 0 else 0.0
                        dh = x[k, c, f, 1, w] - x[k, c, f, 0, w] if h == 0 else 0.0
                        dw = x[k, c, f, h, 1] - x[k, c, f, h, 0] if w == 0 else 0.0
                        total += d2 + 0.5 * abs(df) + 0.5 * math.hypot(dh, dw)
    got = oracle.block_scores(lat, (2, 2, 2))
    assert got[0] == pytest.approx(total / (2 * 2 * 8), rel=1e-13)


# ---------------------------------------------------------------- o2 classify
def test_classify_hand_example():
    g = golden("classify_hand.json")
    s = np.array(g["scores"], dtype=np.float32)
    for case in g["cases"]:
        got = oracle.classify(s, case["frac_active"], case["frac_static"])
        np.testing.assert_array_equal(got, case["levels"])


def _levels_by_counting(scores, nA, nS):
    # rank = number of blocks strictly before in (score, index) order
    B = len(scores)
    out = np.empty(B, dtype=np.uint8)
    for i in range(B):
        r = sum(1 for j in range(B) if (scores[j] < scores[i]) or (scores[j] == scores[i] and j < i))
        out[i] = 1 if r < nS else (3 if r >= B - nA else 2)
    return out


@pytest.mark.parametrize("B", [1, 2, 3, 5, 8])
def test_classify_brute_force_with_ties(B):
    gen = np.random.default_rng(100 + B)
    for trial in range(30):
        s = gen.choice(np.array([-1.0, 0.0, 0.5, 0.5, 2.0], dtype=np.float32), size=B)
        fa, fs = gen.choice([0.0, 0.1, 0.25, 0.3, 0.5]), gen.choice([0.0, 0.2, 0.4, 0.5])
        nA, nS = math.floor(round(fa * 10000) * B / 10000), math.floor(round(fs * 10000) * B / 10000)
        assert oracle.level_counts(B, fa, fs) == (nA, nS)
        np.testing.assert_array_equal(oracle.classify(s, fa, fs), _levels_by_counting(s, nA, nS))


def test_classify_matches_lexsort_and_counts():
    gen = np.random.default_rng(7)
    s = gen.standard_normal(5000).astype(np.float32)
    s[::7] = s[3]                       # many ties
    lv = oracle.classify(s, 0.25, 0.45)
    order = np.lexsort((np.arange(s.size), s.astype(np.float64)))
    nA, nS = 1250, 2250
    expect = np.full(s.size, 2, dtype=np.uint8)
    expect[order[:nS]] = 1
    expect[order[s.size - nA:]] = 3
    np.testing.assert_array_equal(lv, expect)
    assert (lv == 3).sum() == nA and (lv == 1).sum() == nS
    # monotone: every Active score >= every Moderate score >= every Static score
    assert s[lv == 3].min() >= s[lv == 2].max()
    assert s[lv == 2].min() >= s[lv == 1].max()


def test_classify_all_equal_scores_split_by_index():
    lv = oracle.classify(np.zeros(10, dtype=np.float32), 0.3, 0.3)
    np.testing.assert_array_equal(lv, [1, 1, 1, 2, 2, 2, 2, 3, 3, 3])


def test_classify_count_rounding_of_fractions():
    # 0.45f is 0.449999988...; the split counts whole basis points
    assert oracle.level_counts(75600, 0.25, 0.45) == (18900, 34020)
    assert oracle.level_counts(4096, 0.3, 0.4) == (1228, 1638)
    assert oracle.level_counts(32760, 0.35, 0.65) == (11466, 21294)


def test_classify_rejects_bad_input():
    with pytest.raises(oracle.OracleError) as e:
        oracle.classify(np.array([0.0, np.nan], dtype=np.float32), 0.5, 0.0)
    assert e.value.code == oracle.ENONFINITE
    with pytest.raises(oracle.OracleError):
        oracle.classify(np.array([0.0, np.inf], dtype=np.float32), 0.5, 0.0)
    with pytest.raises(oracle.OracleError) as e:
        oracle.classify(np.zeros(4, dtype=np.float32), 0.6, 0.6)
    assert e.value.code == oracle.EINVAL


# ---------------------------------------------------------------- o3 schedule
def test_schedule_hand_example():
    g = golden("schedule_hand.json")
    off, idx, tl = oracle.build_schedule(
        np.array(g["block_levels"], dtype=np.uint8), g["dims"], g["block"], g["patch"],
        g["T"], g["warmup"], g["cooldown"], g["period_moderate"], g["period_static"])
    np.testing.assert_array_equal(off, g["offsets"])
    np.testing.assert_array_equal(idx, g["idx"])


def test_token_map_hand_example():
    g = golden("token_map_hand.json")
    _, _, tl = oracle.build_schedule(np.array(g["block_levels"], dtype=np.uint8),
                                     g["dims"], g["block"], g["patch"], 1, 1, 0, 1, 1)
    np.testing.assert_array_equal(tl, g["token_levels"])


def test_token_map_equals_upsampling():
    # blocks of 1x4x4 latent = 2x2 tokens of 1x2x2: token levels are the block
    # levels repeated twice along th and tw (numpy repeat)
    gen = np.random.default_rng(3)
    F, H, W = 3, 16, 24
    bl = gen.integers(1, 4, size=(F, 4, 6)).astype(np.uint8)
    _, _, tl = oracle.build_schedule(bl.ravel(), (F, H, W), (1, 4, 4), (1, 2, 2), 1, 1, 0, 1, 1)
    expect = bl.repeat(2, axis=1).repeat(2, axis=2)
    np.testing.assert_array_equal(tl, expect.ravel())


def test_schedule_closed_form_counts_50_steps():
    # 50 steps, warm-up 5, cool-down 5, Moderate every 2, Static every 4:
    # per token Active 40 + 10, Moderate 20 + 10, Static 10 + 10 refreshes.
    w = synth.WORKLOADS["schedule50"]
    TF, TH, TW = w.grid
    gen = np.random.default_rng(0)
    bl = gen.integers(1, 4, size=TF * TH * TW).astype(np.uint8)
    off, idx, tl = oracle.build_schedule(bl, (w.F, w.H, w.W), w.block, w.patch, w.T,
                                         w.warmup, w.cooldown, w.period_moderate, w.period_static)
    nA, nM, nS = (bl == 3).sum(), (bl == 2).sum(), (bl == 1).sum()
    N = bl.size
    assert off[-1] == 10 * N + 40 * nA + 20 * nM + 10 * nS
    counts = np.bincount(idx, minlength=N)
    np.testing.assert_array_equal(counts[bl == 3], 50)
    np.testing.assert_array_equal(counts[bl == 2], 30)
    np.testing.assert_array_equal(counts[bl == 1], 20)
    per_step = np.diff(off)
    assert np.all(per_step[:5] == N) and np.all(per_step[-5:] == N)
    # three kinds of interleaved steps
    assert sorted(set(per_step[5:-5].tolist())) == sorted({nA, nA + nM, nA + nM + nS})


def test_schedule_lists_sorted_and_refresh_gaps():
    w = synth.WORKLOADS["schedule50"]
    gen = np.random.default_rng(1)
    N = 600
    bl = gen.integers(1, 4, size=N).astype(np.uint8)
    pM, pS = 3, 5
    off, idx, _ = oracle.build_schedule(bl, (1, 1, N), (1, 1, 1), (1, 1, 1), 40, 4, 3, pM, pS)
    last = np.full(N, -1)
    for s in range(40):
        lst = idx[off[s]:off[s + 1]]
        assert np.all(np.diff(lst) > 0) and (lst.size == 0 or (lst[0] >= 0 and lst[-1] < N))
        if 4 <= s < 37:
            # no token waits more than its period between refreshes
            gap = s - last
            assert np.all(gap[bl == 3] == 1)
            assert np.all(gap[bl == 2] <= pM)
            assert np.all(gap[bl == 1] <= pS)
        last[lst] = s


# ---------------------------------------------------------------- o4 scatter
def test_kv_scatter_matches_numpy_indexing():
    gen = np.random.default_rng(9)
    N, H, d = 257, 3, 64
    kc = gen.integers(0, 65535, size=(N, H, d), dtype=np.uint16)
    vc = gen.integers(0, 65535, size=(N, H, d), dtype=np.uint16)
    idx = np.sort(gen.choice(N, size=77, replace=False)).astype(np.int32)
    ka = gen.integers(0, 65535, size=(77, H, d), dtype=np.uint16)
    va = gen.integers(0, 65535, size=(77, H, d), dtype=np.uint16)
    k2, v2 = oracle.kv_scatter(ka, va, idx, kc, vc)
    ek, ev = kc.copy(), vc.copy()
    ek[idx] = ka
    ev[idx] = va
    np.testing.assert_array_equal(k2, ek)
    np.testing.assert_array_equal(v2, ev)
    untouched = np.setdiff1d(np.arange(N), idx)
    np.testing.assert_array_equal(k2[untouched], kc[untouched])


def test_kv_scatter_rejects_out_of_range_index():
    z = np.zeros((4, 1, 8), dtype=np.uint16)
    with pytest.raises(oracle.OracleError) as e:
        oracle.kv_scatter(z[:1], z[:1], np.array([4], dtype=np.int32), z, z)
    assert e.value.code == oracle.EINDEX


# ---------------------------------------------------------------- o5 attention
def _sdpa64(q, k, v, scale):
    import torch
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]      # [1, H, n, d]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_hand_example():
    g = golden("attention_hand.json")
    q = synth.bf16_bits(np.array(g["q"], dtype=np.float32))
    k = synth.bf16_bits(np.array(g["k_cache"], dtype=np.float32))
    v = synth.bf16_bits(np.array(g["v_cache"], dtype=np.float32))
    out = oracle.active_attention(q, k, v, scale=g["scale"])
    np.testing.assert_allclose(out, g["expected"], rtol=1e-14)


def test_attention_all_active_equals_full_attention():
    gen = np.random.default_rng(21)
    N, H, d = 48, 3, 16
    q, k, v = (synth.bf16_normal((N, H, d), gen) for _ in range(3))
    out = oracle.active_attention(q, k, v)
    ref = _sdpa64(*(synth.bf16_to_f32(a).astype(np.float64) for a in (q, k, v)), 1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_attention_fresh_cache_equals_rows_of_full_attention():
    gen = np.random.default_rng(22)
    N, H, d = 64, 2, 32
    q, k, v = (synth.bf16_normal((N, H, d), gen) for _ in range(3))
    idx = np.sort(gen.choice(N, size=19, replace=False)).astype(np.int32)
    out = oracle.active_attention(q[idx], k, v)
    ref = _sdpa64(*(synth.bf16_to_f32(a).astype(np.float64) for a in (q, k, v)), 1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref[idx], rtol=1e-12, atol=1e-13)


def test_attention_permutation_invariance_of_cache():
    # concatenating [fresh active ; frozen] K/V equals the token-ordered cache
    gen = np.random.default_rng(23)
    N, H, d = 40, 2, 16
    q = synth.bf16_normal((7, H, d), gen)
    k, v = synth.bf16_normal((N, H, d), gen), synth.bf16_normal((N, H, d), gen)
    act = np.sort(gen.choice(N, size=7, replace=False))
    frozen = np.setdiff1d(np.arange(N), act)
    cat = np.concatenate([act, frozen])
    a = oracle.active_attention(q, k, v)
    b = oracle.active_attention(q, k[cat], v[cat])
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_attention_single_key_and_identical_keys():
    gen = np.random.default_rng(24)
    H, d = 2, 8
    q = synth.bf16_normal((3, H, d), gen)
    k1, v1 = synth.bf16_normal((1, H, d), gen), synth.bf16_normal((1, H, d), gen)
    out = oracle.active_attention(q, k1, v1)
    np.testing.assert_array_equal(out, np.broadcast_to(synth.bf16_to_f32(v1), out.shape))
    kk = np.broadcast_to(synth.bf16_normal((1, H, d), gen), (9, H, d)).copy()
    vv = synth.bf16_normal((9, H, d), gen)
    out = oracle.active_attention(q, kk, vv)
    np.testing.assert_allclose(out, np.broadcast_to(synth.bf16_to_f32(vv).astype(np.float64).mean(0), out.shape),
                               rtol=1e-13, atol=1e-15)


def test_attention_row_selection():
    gen = np.random.default_rng(25)
    q, k, v = (synth.bf16_normal((20, 2, 8), gen) for _ in range(3))
    full = oracle.active_attention(q, k, v)
    rows = np.array([19, 0, 7], dtype=np.int32)
    np.testing.assert_array_equal(oracle.active_attention(q, k, v, rows=rows), full[rows])


# ---------------------------------------------------------------- generators
def test_bf16_rounding_matches_torch():
    import torch
    gen = np.random.default_rng(0)
    x = np.concatenate([gen.standard_normal(10000).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 3.4e38, -1e-40], dtype=np.float32)])
    ours = synth.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


# ---------------------------------------------------------------- projections of the active rows
def _bits(a):
    return synth.bf16_bits(np.asarray(a, dtype=np.float32))


def test_gather_gemm_hand_example():
    g = golden("gather_gemm_hand.json")
    got = oracle.gather_gemm(_bits(g["x"]), _bits(g["w"]), np.array(g["gather"], dtype=np.int32))
    np.testing.assert_array_equal(got, np.array(g["expected"]))


def test_gather_gemm_identity_weight_gathers_rows_exactly():
    gen = np.random.default_rng(31)
    x = synth.bf16_normal((40, 24), gen)
    gather = gen.integers(0, 40, size=17).astype(np.int32)
    eye = _bits(np.eye(24))
    got = oracle.gather_gemm(x, eye, gather)
    np.testing.assert_array_equal(got, synth.bf16_to_f32(x)[gather].astype(np.float64))


def test_gather_gemm_matches_library_matmul():
    # the same product by numpy's fp64 matmul and by torch's fp64 linear layer
    import torch
    gen = np.random.default_rng(32)
    x, w = synth.bf16_normal((50, 72), gen), synth.bf16_normal((30, 72), gen)
    gather = gen.integers(0, 50, size=23).astype(np.int32)
    got = oracle.gather_gemm(x, w, gather)
    xf, wf = synth.bf16_to_f32(x).astype(np.float64), synth.bf16_to_f32(w).astype(np.float64)
    np.testing.assert_allclose(got, xf[gather] @ wf.T, rtol=1e-12, atol=1e-12)
    tl = torch.nn.functional.linear(torch.from_numpy(xf[gather]), torch.from_numpy(wf)).numpy()
    np.testing.assert_allclose(got, tl, rtol=1e-12, atol=1e-12)


def test_gather_gemm_rows_follow_the_gather_and_default_to_identity():
    gen = np.random.default_rng(33)
    x, w = synth.bf16_normal((12, 16), gen), synth.bf16_normal((8, 16), gen)
    full = oracle.gather_gemm(x, w)                       # no gather: row r reads x[r]
    perm = gen.permutation(12).astype(np.int32)
    np.testing.assert_array_equal(oracle.gather_gemm(x, w, perm), full[perm])
    np.testing.assert_array_equal(oracle.gather_gemm(x, w, np.array([5, 5], dtype=np.int32)), full[[5, 5]])


def test_gather_gemm_is_linear_in_the_weight_and_transposes_right():
    # a wrong operand orientation (x @ w instead of x @ w^T) or a dropped
    # term breaks these: one-hot weight rows pick single input columns
    gen = np.random.default_rng(34)
    x = synth.bf16_normal((9, 6), gen)
    onehot = np.zeros((3, 6), dtype=np.float32)
    onehot[0, 5] = 1.0
    onehot[1, 0] = 1.0
    onehot[2, 2] = -2.0
    got = oracle.gather_gemm(x, _bits(onehot))
    xf = synth.bf16_to_f32(x).astype(np.float64)
    np.testing.assert_array_equal(got[:, 0], xf[:, 5])
    np.testing.assert_array_equal(got[:, 1], xf[:, 0])
    np.testing.assert_array_equal(got[:, 2], -2.0 * xf[:, 2])
    w1, w2 = synth.bf16_normal((4, 6), gen), synth.bf16_normal((4, 6), gen)
    both = np.concatenate([w1, w2])
    np.testing.assert_array_equal(oracle.gather_gemm(x, both),
                                  np.concatenate([oracle.gather_gemm(x, w1), oracle.gather_gemm(x, w2)], axis=1))


def test_gather_gemm_rejects_out_of_range_row():
    x = _bits(np.ones((4, 8)))
    with pytest.raises(oracle.OracleError):
        oracle.gather_gemm(x, x, np.array([0, 4], dtype=np.int32))


# ---------------------------------------------------------------- random-masking ablation
def test_splitmix64_known_answers():
    g = golden("splitmix64_seed0.json")
    got = oracle.splitmix64(g["seed"], 4)
    assert [f"{int(v):016x}" for v in got] == g["expected_hex"]


def test_random_scores_follow_the_stream_and_are_uniform():
    n, seed = 200000, 12345
    s = oracle.random_scores(n, seed)
    raw = oracle.splitmix64(seed, n)
    # the score is the top 24 bits of output b+1, exactly
    np.testing.assert_array_equal(s, ((raw >> np.uint64(40)).astype(np.float64) / 2**24).astype(np.float32))
    assert s.min() >= 0.0 and s.max() < 1.0
    # uniform: mean, variance and a 20-bin chi-square (df 19; 60 is far past p = 1e-6)
    assert abs(s.mean() - 0.5) < 5 / math.sqrt(12 * n)
    assert abs(s.var() - 1 / 12) < 0.002
    hist = np.histogram(s, bins=20, range=(0, 1))[0]
    chi2 = ((hist - n / 20) ** 2 / (n / 20)).sum()
    assert chi2 < 60
    # another seed gives another stream
    assert not np.array_equal(s[:100], oracle.random_scores(100, seed + 1))


def test_random_level_map_keeps_the_level_counts():
    # the ablation assigns Jano's level counts at random: same n_A / n_S
    n = 19320
    lv = oracle.classify(oracle.random_scores(n, 7), 0.25, 0.45)
    n_a, n_s = oracle.level_counts(n, 0.25, 0.45)
    assert (lv == 3).sum() == n_a and (lv == 1).sum() == n_s and (lv == 2).sum() == n - n_a - n_s


def test_schedule_closed_form_counts_static_every_5th_step():
    # the page's example period for Level 1 ("e.g. every 5th step"): 50 steps,
    # warm-up 5, cool-down 5, Moderate every 2, Static every 5 -> per token
    # Active 40 + 10, Moderate 20 + 10, Static 8 + 10 refreshes
    gen = np.random.default_rng(5)
    bl = gen.integers(1, 4, size=6 * 7).astype(np.uint8)
    off, idx, tl = oracle.build_schedule(bl, (1, 12, 14), (1, 2, 2), (1, 2, 2), 50, 5, 5, 2, 5)
    counts = np.bincount(idx, minlength=bl.size)
    np.testing.assert_array_equal(counts[bl == 3], 50)
    np.testing.assert_array_equal(counts[bl == 2], 30)
    np.testing.assert_array_equal(counts[bl == 1], 18)


# ---------------------------------------------------------------- literal score reading
def _grad(x, axis):
    """Forward difference along `axis`, 0 at the last index (numpy)."""
    g = np.zeros_like(x)
    sl_lo = [slice(None)] * x.ndim
    sl_hi = [slice(None)] * x.ndim
    sl_lo[axis] = slice(0, -1)
    sl_hi[axis] = slice(1, None)
    g[tuple(sl_lo)] = x[tuple(sl_hi)] - x[tuple(sl_lo)]
    return g


def test_literal_score_equals_gradients_of_the_second_difference():
    # Delta2 and the forward differences are linear and commute, so the
    # literal score (gradients first, then the second difference over steps)
    # equals the gradient magnitudes of the second difference, computed here
    # by numpy in the other order and reduced per block by reshaping
    gen = np.random.default_rng(41)
    lat = gen.standard_normal((5, 3, 4, 8, 12)).astype(np.float32)
    x = lat.astype(np.float64)
    d2 = x[2:] - 2 * x[1:-1] + x[:-2]                        # [K-1][C][F][H][W]
    term = 0.5 * np.abs(_grad(d2, 2)) + 0.5 * np.sqrt(_grad(d2, 3) ** 2 + _grad(d2, 4) ** 2)
    per = term.reshape(3, 3, 4, 2, 4, 3, 4).transpose(2, 3, 5, 0, 1, 4, 6).reshape(4 * 2 * 3, -1)
    np.testing.assert_allclose(oracle.block_scores_literal(lat, (1, 4, 4)), per.mean(axis=1), rtol=1e-12)


def test_literal_score_is_zero_for_steps_affine_in_k():
    # x_k = a(p) + k b(p): every gradient is affine in k, its second difference 0
    gen = np.random.default_rng(42)
    a, b = gen.standard_normal((2, 2, 3, 8, 8))
    lat = np.stack([a + k * b for k in range(6)]).astype(np.float32)
    np.testing.assert_allclose(oracle.block_scores_literal(lat, (1, 4, 4)), 0.0, atol=2e-5)


def test_literal_score_closed_forms_for_quadratic_steps():
    # x_k = k^2 c(p): Delta2 of any gradient of x is 2 * (gradient of c).
    # c = alpha * h: spatial term 2|alpha| except the last row (0);
    # c = beta * f: temporal term 2|beta| except the last frame (0)
    K1, F, H, W = 5, 3, 8, 8
    alpha, beta = 0.75, -1.25
    hh = np.arange(H, dtype=np.float64)[None, None, :, None] * np.ones((1, F, 1, W))
    ff = np.arange(F, dtype=np.float64)[None, :, None, None] * np.ones((1, 1, H, W))
    for c_field, expect in ((alpha * hh, "h"), (beta * ff, "f")):
        lat = np.stack([k * k * c_field for k in range(K1)]).astype(np.float32)
        got = oracle.block_scores_literal(lat, (1, 4, 4), 0.5, 0.5).reshape(F, 2, 2)
        if expect == "h":
            # rows 0..3 of block row 0 all interior; block row 1 has rows 4..7, row 7 is the edge
            np.testing.assert_allclose(got[:, 0, :], 0.5 * 2 * abs(alpha), rtol=1e-6)
            np.testing.assert_allclose(got[:, 1, :], 0.5 * 2 * abs(alpha) * 3 / 4, rtol=1e-6)
        else:
            np.testing.assert_allclose(got[:-1], 0.5 * 2 * abs(beta), rtol=1e-6)
            np.testing.assert_allclose(got[-1], 0.0, atol=1e-12)


def test_literal_and_additive_readings_differ():
    # the two readings are different scores (the additive one has |Delta2 x|
    # and first-order gradients): a plain spatial ramp constant over the steps
    # scores 0 under the literal reading but not under the additive one
    hh = np.arange(8, dtype=np.float32)[None, None, None, :, None] * np.ones((6, 1, 2, 8, 8), np.float32)
    assert np.all(oracle.block_scores_literal(hh, (1, 4, 4)) == 0.0)
    assert np.all(oracle.block_scores(hh, (1, 4, 4))[:2] > 0.0)


# ---------------------------------------------------------------- FFT baseline score
def _blocks(x, block):
    """Yield (block index, [C][mf][mh][mw] view) in block order."""
    Cc, F, H, W = x.shape
    bf, bh, bw = block
    b = 0
    for f0 in range(0, F, bf):
        for h0 in range(0, H, bh):
            for w0 in range(0, W, bw):
                yield b, x[:, f0:f0 + bf, h0:h0 + bh, w0:w0 + bw].astype(np.float64)
                b += 1


def _ragged_snapshot(seed):
    # partial blocks on every axis for the (2, 4, 4) blocks
    return np.random.default_rng(seed).standard_normal((3, 5, 10, 13)).astype(np.float32) * 1.5 + 0.3


@pytest.mark.parametrize("block", [(1, 4, 4), (2, 4, 4), (1, 2, 2), (3, 3, 5)])
def test_fft_score_cutoff0_is_the_mean_square_by_parseval(block):
    x = _ragged_snapshot(1)
    s = oracle.fft_scores(x, block, 0)
    for b, blk in _blocks(x, block):
        want = np.mean([np.mean(blk[c] ** 2) for c in range(x.shape[0])])
        assert s[b] == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("block", [(1, 4, 4), (2, 4, 4), (1, 2, 2), (3, 3, 5)])
def test_fft_score_cutoff1_is_the_block_variance_by_parseval(block):
    # everything but the DC bin: the population variance of each channel's block
    x = _ragged_snapshot(2)
    s = oracle.fft_scores(x, block, 1)
    for b, blk in _blocks(x, block):
        want = np.mean([np.var(blk[c]) for c in range(x.shape[0])])
        assert s[b] == pytest.approx(want, rel=1e-10, abs=1e-13)


@pytest.mark.parametrize("block,cutoff", [((1, 4, 4), 2), ((2, 4, 4), 1), ((2, 4, 4), 2), ((3, 3, 5), 2),
                                          ((1, 8, 8), 3)])
def test_fft_score_matches_library_fft_per_block(block, cutoff):
    x = np.random.default_rng(3).standard_normal((2, 4, 17, 19)).astype(np.float32)
    s = oracle.fft_scores(x, block, cutoff)
    for b, blk in _blocks(x, block):
        m = blk.shape[1:]
        fold = [np.abs(np.fft.fftfreq(n) * n).round().astype(int) for n in m]
        kmax = np.maximum.reduce(np.meshgrid(*fold, indexing="ij"))
        e = [np.sum(np.abs(np.fft.fftn(blk[c])) ** 2 * (kmax >= cutoff)) for c in range(blk.shape[0])]
        want = np.mean(e) / np.prod(m) ** 2
        assert s[b] == pytest.approx(want, rel=1e-10, abs=1e-14)


def test_fft_score_planted_frequencies():
    # a cosine of one cycle per block along h: energy a^2/2, all at folded
    # index 1; the Nyquist pattern (-1)^h: energy a^2 at folded index 2
    a = 1.75
    h = np.arange(8)
    cos1 = np.broadcast_to((a * np.cos(2 * np.pi * h / 4))[None, None, :, None], (1, 1, 8, 8)).astype(np.float32)
    nyq = np.broadcast_to((a * (-1.0) ** h)[None, None, :, None], (1, 1, 8, 8)).astype(np.float32)
    for cutoff, want in ((0, a * a / 2), (1, a * a / 2), (2, 0.0)):
        np.testing.assert_allclose(oracle.fft_scores(cos1, (1, 4, 4), cutoff), want, atol=1e-12)
    for cutoff, want in ((1, a * a), (2, a * a), (3, 0.0)):
        np.testing.assert_allclose(oracle.fft_scores(nyq, (1, 4, 4), cutoff), want, atol=1e-12)


def test_fft_score_cutoff_above_every_index_is_zero_and_scores_are_ordered():
    x = _ragged_snapshot(4)
    s = [oracle.fft_scores(x, (2, 4, 4), k) for k in range(4)]
    assert np.all(s[3] == 0.0)
    for lo, hi in zip(s, s[1:]):
        assert np.all(hi <= lo + 1e-12)          # a higher cutoff keeps fewer bins
