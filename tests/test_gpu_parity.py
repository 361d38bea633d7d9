"""GPU (sm_100a) parity against the fp64 CPU oracle, through the C ABI.

Bit-exact: level maps, schedules (offsets, index lists, token levels) and
the KV-cache scatter.  Floating point: block scores within
|gpu - ref| <= 1e-5 |ref| + 1e-7 (fp32 accumulation), attention outputs
within max-abs 2e-2 and mean-rel 5e-3 (sum|gpu-ref| / sum|ref|) of the fp64
values (BF16 in and out, fp32 accumulation and softmax).

Every workload of the benchmark set runs at its full size.  Attention on the
two video workloads is compared on sampled rows, since the oracle takes up to
a second per row there: at least 256 rows chosen so that every position of
the kernel's grid is reached (both query tiles of a CTA's pair, all four
32-row TMEM lane quarters, the first, last and evenly spaced CTAs, the
ragged last pair), all heads of each row.  The oracle rows run concurrently
on the host cores.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from workloads import (attention_case, attention_errors, cta_position_rows, latent,
                       oracle_attention_rows, sample_rows, token_field, token_geometry)

pytestmark = pytest.mark.gpu

ATT_MAX_ABS = 2e-2
ATT_MEAN_REL = 5e-3
SCORE_RTOL, SCORE_ATOL = 1e-5, 1e-7
ALL = ["tiny", "image", "small", "large"]


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


def dev_bf16(t):
    return t.contiguous().to("cuda")


def host_bits(t):
    return synth.bits_of(t.cpu())


def no_device_error(J):
    code = J.device_error()
    assert code == 0, J.jano_status_str(code)


# ---------------------------------------------------------------- analyzer
@pytest.mark.parametrize("name", ALL)
def test_block_scores_match_oracle(J, name):
    w = synth.WORKLOADS[name]
    lat = latent(name)
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    got = J.block_scores(torch.from_numpy(lat).cuda(), geom).cpu().numpy()
    ref = oracle.block_scores(lat, w.block)
    no_device_error(J)
    assert got.shape == ref.shape
    np.testing.assert_array_less(np.abs(got - ref), SCORE_RTOL * np.abs(ref) + SCORE_ATOL)
    # deterministic: a second launch gives the same bits
    again = J.block_scores(torch.from_numpy(lat).cuda(), geom).cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), again.view(np.uint32))


@pytest.mark.parametrize("shape,block", [((3, 2, 3, 9, 12), (1, 4, 4)),     # partial rows/cols
                                         ((4, 3, 5, 6, 8), (2, 3, 2)),      # bf > 1, odd blocks
                                         ((6, 1, 1, 16, 16), (1, 2, 2)),    # F = 1
                                         ((3, 1, 2, 4, 20), (1, 4, 8)),     # bw = 8, partial
                                         ((4, 3, 3, 9, 520), (1, 4, 4)),    # wide rows: boxed chunks
                                         ((3, 2, 2, 6, 200), (2, 4, 8)),    # whole rows, bf = 2
                                         # K = 5, blocks of one frame (the frame-group form):
                                         ((6, 2, 1, 9, 20), (1, 4, 4)),     # F = 1, partial row, odd blocks
                                         ((6, 3, 5, 14, 200), (1, 4, 4)),   # several column chunks, ragged
                                         ((6, 2, 11, 8, 328), (1, 4, 4)),   # frame groups, wide rows
                                         ((6, 1, 21, 6, 48), (1, 4, 4)),    # many frame groups, short rows
                                         ((6, 2, 7, 13, 52), (1, 4, 4)),    # ragged H, W and last frame group
                                         ((6, 3, 5, 10, 96), (1, 2, 8)),    # bh = 2, bw = 8
                                         ((6, 2, 4, 9, 40), (1, 1, 1)),     # one-element blocks
                                         ((6, 2, 3, 7, 200), (1, 4, 32)),   # bw = 32, ragged last block
                                         ((6, 2, 9, 6, 36), (1, 2, 16)),    # bw = 16, ragged last block
                                         ((6, 2, 2, 5, 4), (1, 4, 4)),      # one float4 per row
                                         ((6, 2, 3, 11, 24), (1, 2, 2))])   # 2x2 blocks, ragged rows
def test_block_scores_edge_geometries(J, shape, block):
    g = np.random.default_rng(sum(shape))
    lat = g.standard_normal(shape).astype(np.float32)
    K1, Cc, F, H, W = shape
    geom = J.Geometry(F, H, W, block, (1, 1, 1))
    got = J.block_scores(torch.from_numpy(lat).cuda(), geom).cpu().numpy()
    ref = oracle.block_scores(lat, block)
    np.testing.assert_array_less(np.abs(got - ref), SCORE_RTOL * np.abs(ref) + SCORE_ATOL)


def test_block_scores_constant_latent_is_zero(J):
    lat = torch.full((6, 16, 4, 32, 32), 3.25, device="cuda")
    got = J.block_scores(lat, J.Geometry(4, 32, 32))
    assert torch.all(got == 0)


# ---------------------------------------------------------------- classify
@pytest.mark.parametrize("name", ALL)
def test_classify_token_field_bit_exact(J, name):
    w = synth.WORKLOADS[name]
    field = token_field(w)
    got = J.classify(torch.from_numpy(field).cuda(), w.frac_active, w.frac_static).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.classify(field, w.frac_active, w.frac_static))


@pytest.mark.parametrize("name", ALL)
def test_classify_gpu_scores_bit_exact_and_end_to_end(J, name):
    w = synth.WORKLOADS[name]
    lat = latent(name)
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    s_gpu = J.block_scores(torch.from_numpy(lat).cuda(), geom)
    lv_gpu = J.classify(s_gpu, w.frac_active, w.frac_static).cpu().numpy()
    s_host = s_gpu.cpu().numpy()
    # stage-wise: both classify the same fp32 scores
    np.testing.assert_array_equal(lv_gpu, oracle.classify(s_host, w.frac_active, w.frac_static))
    # end to end: oracle scores (rounded to fp32) -> oracle levels; report flips
    lv_ref = oracle.classify(oracle.block_scores(lat, w.block).astype(np.float32), w.frac_active,
                             w.frac_static)
    flips = int((lv_ref != lv_gpu).sum())
    print(f"{name}: end-to-end level flips {flips} of {lv_gpu.size}")
    assert flips <= max(2, lv_gpu.size // 1000)


@pytest.mark.parametrize("n", [1, 2, 7, 1023, 1024, 1025, 5000, 100_003, 400_003])
def test_classify_ties_and_sizes(J, n):
    g = np.random.default_rng(n)
    s = g.choice(np.array([-2.0, -0.0, 0.0, 0.5, 0.5, 1.0, 3.0], dtype=np.float32), size=n)
    for fa, fs in [(0.3, 0.4), (0.0, 0.0), (1.0, 0.0), (0.0, 1.0), (0.25, 0.45), (0.5, 0.5)]:
        got = J.classify(torch.from_numpy(s).cuda(), fa, fs).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.classify(s, fa, fs), err_msg=f"{fa},{fs}")


@pytest.mark.parametrize("dist", ["normal", "outliers", "lognormal", "denormal", "narrow", "mixed_sign_zero"])
def test_classify_value_domain_first_pass(J, dist):
    # the first pass bins float values: few candidates (direct rank), crowded
    # bins (radix over the gathered candidates) and bins beyond the gather
    # buffers (the select starts over on the order keys), all against the oracle
    g = np.random.default_rng(len(dist))
    n = 75_600
    if dist == "normal":
        s = g.standard_normal(n)
    elif dist == "outliers":                        # a few huge values: one bin holds almost all
        s = g.standard_normal(n)
        s[g.choice(n, 5, replace=False)] = [1e30, -1e30, 3e29, 1e25, -7e28]
    elif dist == "lognormal":
        s = g.lognormal(0.0, 4.0, n)
    elif dist == "denormal":                        # subnormal floats only
        s = g.integers(1, 1 << 20, n).astype(np.uint32).view(np.float32).astype(np.float64)
    elif dist == "narrow":                          # a handful of distinct floats near 1
        s = 1.0 + g.integers(0, 40, n) * 2.0 ** -23
    else:                                           # signed zeros and small integers
        s = g.choice([-0.0, 0.0, -1.0, 1.0, 2.0], n) + g.choice([0.0, 0.25], n)
    s = s.astype(np.float32)
    for fa, fs in [(0.25, 0.45), (0.3, 0.4), (0.0, 0.5), (0.5, 0.0), (0.01, 0.98)]:
        got = J.classify(torch.from_numpy(s).cuda(), fa, fs).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.classify(s, fa, fs), err_msg=f"{dist} {fa},{fs}")


def test_classify_all_equal_split_by_index(J):
    got = J.classify(torch.zeros(10, device="cuda"), 0.3, 0.3).cpu().numpy()
    np.testing.assert_array_equal(got, [1, 1, 1, 2, 2, 2, 2, 3, 3, 3])


def test_classify_non_finite_sets_device_error(J):
    s = torch.tensor([0.0, float("nan"), 1.0], device="cuda")
    J.classify(s, 0.3, 0.3)
    assert J.device_error() == 5
    assert J.device_error() == 0        # read-and-clear


# ---------------------------------------------------------------- schedule
def _schedule_both(J, levels, dims, block, patch, sched):
    geom = J.Geometry(*dims, block, patch)
    off, idx, tl = J.build_schedule(torch.from_numpy(levels).cuda(), geom, sched)
    off = off.cpu().numpy()
    idx = idx.cpu().numpy()[: off[-1]]
    tl = tl.cpu().numpy()
    r_off, r_idx, r_tl = oracle.build_schedule(levels, dims, block, patch, sched.T, sched.warmup,
                                               sched.cooldown, sched.period_moderate,
                                               sched.period_static)
    np.testing.assert_array_equal(off, r_off)
    np.testing.assert_array_equal(idx, r_idx)
    np.testing.assert_array_equal(tl, r_tl)
    return off, idx


@pytest.mark.parametrize("name", ALL + ["schedule50"])
def test_schedule_bit_exact(J, name):
    w = synth.WORKLOADS[name]
    sched = J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static)
    # token-field levels, every token its own block
    field = token_field(w)
    lv = oracle.classify(field, w.frac_active, w.frac_static)
    _schedule_both(J, lv, *token_geometry(w), sched)
    # analyzer blocks mapped onto tokens
    g = np.random.default_rng(w.seed)
    blv = g.integers(1, 4, size=w.n_blocks).astype(np.uint8)
    _schedule_both(J, blv, (w.F, w.H, w.W), w.block, w.patch, sched)
    no_device_error(J)


@pytest.mark.parametrize("cfg", [(1, 1, 0, 1, 1), (7, 7, 0, 2, 3), (10, 0, 0, 1, 1),
                                 (12, 2, 3, 5, 2), (40, 4, 3, 3, 5)])
def test_schedule_configs(J, cfg):
    g = np.random.default_rng(sum(cfg))
    lv = g.integers(1, 4, size=3 * 5 * 7).astype(np.uint8)
    _schedule_both(J, lv, (3, 10, 14), (1, 2, 2), (1, 2, 2), J.Schedule(*cfg))


def test_schedule_bad_level_sets_device_error(J):
    lv = np.array([1, 2, 9, 3], dtype=np.uint8)
    J.build_schedule(torch.from_numpy(lv).cuda(), J.Geometry(1, 1, 4, (1, 1, 1), (1, 1, 1)),
                     J.Schedule(3, 1, 1, 1, 1))
    assert J.device_error() == 6


# ---------------------------------------------------------------- KV scatter
@pytest.mark.parametrize("name", ALL)
def test_kv_scatter_bit_exact(J, name):
    c = attention_case(name)
    idx = c["idx"]
    kc, vc = dev_bf16(c["k_stale"]), dev_bf16(c["v_stale"])
    J.kv_scatter(dev_bf16(c["k_act"]), dev_bf16(c["v_act"]), torch.from_numpy(idx).cuda(), kc, vc)
    no_device_error(J)
    rk, rv = oracle.kv_scatter(synth.bits_of(c["k_act"]), synth.bits_of(c["v_act"]), idx,
                               synth.bits_of(c["k_stale"]), synth.bits_of(c["v_stale"]))
    np.testing.assert_array_equal(host_bits(kc), rk)
    np.testing.assert_array_equal(host_bits(vc), rv)


def test_kv_scatter_odd_rows_and_bad_index(J):
    g = np.random.default_rng(3)
    N, H, d = 50, 3, 64
    kc = torch.randn(N, H, d, device="cuda").bfloat16()
    vc = torch.randn(N, H, d, device="cuda").bfloat16()
    before_k, before_v = kc.clone(), vc.clone()
    idx = np.array([0, 5, 17, 49, 50], dtype=np.int32)      # 50 is out of range
    ka = torch.randn(5, H, d, device="cuda").bfloat16()
    va = torch.randn(5, H, d, device="cuda").bfloat16()
    J.kv_scatter(ka, va, torch.from_numpy(idx).cuda(), kc, vc)
    assert J.device_error() == 6
    ok = [0, 1, 2, 3]
    assert torch.equal(kc[idx[ok]], ka[ok]) and torch.equal(vc[idx[ok]], va[ok])
    rest = np.setdiff1d(np.arange(N), idx[ok])
    assert torch.equal(kc[rest], before_k[rest]) and torch.equal(vc[rest], before_v[rest])


# ---------------------------------------------------------------- attention
def _attention_check(J, q, kc, vc, idx, rows, scale=None):
    """Run the GPU kernel on (q, kc, vc, idx); compare the sampled rows."""
    N, H, d = kc.shape
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(idx).cuda(), out,
                       scale=scale)
    no_device_error(J)
    got = out.cpu()
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(kc), synth.bits_of(vc),
                                  scale=scale, rows=rows)
    g = got[torch.from_numpy(idx[rows]).long()].float().numpy()
    mx, mr = attention_errors(g, ref)
    # rows not in idx stay untouched (zero)
    mask = torch.ones(N, dtype=torch.bool)
    mask[torch.from_numpy(idx).long()] = False
    assert torch.count_nonzero(got[mask].float()) == 0
    return mx, mr, out


def attention_rows_for(name, n_act, seed):
    """All rows for tiny; grid-position rows (>= 256) plus seeded random ones
    for the others."""
    if name == "tiny":
        return np.arange(n_act, dtype=np.int32)
    pos = cta_position_rows(n_act, n_ctas=32, seed=seed)
    extra = sample_rows(n_act, 256 if pos.size < 256 else 64, seed=seed + 1)
    rows = np.unique(np.concatenate([pos, extra])).astype(np.int32)
    assert rows.size >= min(256, n_act)
    return rows


@pytest.mark.parametrize("name", ALL)
def test_attention_after_scatter_matches_oracle(J, name):
    c = attention_case(name)
    w, idx = c["w"], c["idx"]
    kc, vc = dev_bf16(c["k_stale"]), dev_bf16(c["v_stale"])
    J.kv_scatter(dev_bf16(c["k_act"]), dev_bf16(c["v_act"]), torch.from_numpy(idx).cuda(), kc, vc)
    # the oracle's inputs come from the oracle's own scatter of the same rows
    rk, rv = oracle.kv_scatter(synth.bits_of(c["k_act"]), synth.bits_of(c["v_act"]), idx,
                               synth.bits_of(c["k_stale"]), synth.bits_of(c["v_stale"]))
    rows = attention_rows_for(name, idx.size, w.seed)
    N, H, d = kc.shape
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(dev_bf16(c["q_act"]), kc, vc, torch.from_numpy(idx).cuda(), out)
    no_device_error(J)
    ref = oracle_attention_rows(synth.bits_of(c["q_act"]), rk, rv, rows)
    got = out.cpu()
    g = got[torch.from_numpy(idx[rows]).long()].float().numpy()
    mx, mr = attention_errors(g, ref)
    print(f"{name}: rows {rows.size}, max-abs {mx:.3e}, mean-rel {mr:.3e}")
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL
    # per row as well: no single row may be far off while the mean hides it
    per_row = np.abs(g - ref).reshape(rows.size, -1).max(axis=1)
    assert per_row.max() <= ATT_MAX_ABS
    # rows not in idx stay untouched (zero)
    mask = torch.ones(N, dtype=torch.bool)
    mask[torch.from_numpy(idx).long()] = False
    assert torch.count_nonzero(got[mask].float()) == 0


@pytest.mark.parametrize("N,n_act,H,d", [(1, 1, 1, 128), (127, 5, 2, 64), (129, 129, 1, 128),
                                         (1000, 300, 3, 128), (1000, 300, 3, 64),
                                         (384, 256, 2, 128), (2049, 1, 1, 64)])
def test_attention_ragged_shapes(J, N, n_act, H, d):
    g = np.random.default_rng(N * 7 + n_act)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.normal_bf16((n_act, H, d), N + 1)
    kc = synth.normal_bf16((N, H, d), N + 2)
    vc = synth.normal_bf16((N, H, d), N + 3)
    mx, mr, _ = _attention_check(J, q, kc, vc, idx, np.arange(n_act, dtype=np.int32))
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL, (mx, mr)


def test_attention_all_active_is_full_attention(J):
    N, H, d = 777, 2, 128
    q = synth.normal_bf16((N, H, d), 11)
    k = synth.normal_bf16((N, H, d), 12)
    v = synth.normal_bf16((N, H, d), 13)
    idx = np.arange(N, dtype=np.int32)
    mx, mr, out = _attention_check(J, q, k, v, idx, np.arange(N, dtype=np.int32))
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL
    # and against torch's own fp32 attention on the same BF16 inputs
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.float().permute(1, 0, 2)[None], k.float().permute(1, 0, 2)[None],
        v.float().permute(1, 0, 2)[None])[0].permute(1, 0, 2)
    diff = (out.cpu().float() - ref).abs()
    assert float(diff.sum() / ref.abs().sum()) <= ATT_MEAN_REL


def test_attention_peaked_softmax_and_scale(J):
    # Large logits exercise the lazy rescale (running max grows by > 2^8).
    # Outputs here reach |o| ~ 4-8, where the BF16 output rounding alone is
    # up to 2^-8 |o| (BF16 keeps 8 significant bits, unit roundoff 2^-8), so
    # the configs' absolute 2e-2 does not apply; the bound is the
    # arithmetic's: P rounded to BF16 moves o by at most 2^-8 max|v|, the
    # BF16 output rounding by at most 2^-8 |o|.
    N, H, d, n_act = 600, 2, 64, 130
    g = np.random.default_rng(5)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.tensor_of(synth.bf16_bits((3.0 * g.standard_normal((n_act, H, d))).astype(np.float32)))
    base = 3.0 * g.standard_normal((N, H, d)) * np.linspace(0.2, 2.0, N)[:, None, None]
    k = synth.tensor_of(synth.bf16_bits(base.astype(np.float32)))
    v = synth.normal_bf16((N, H, d), 9)
    vmax = float(v.float().abs().amax())
    for scale in (None, 0.5):
        out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
        J.active_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(idx).cuda(), out,
                           scale=scale)
        no_device_error(J)
        ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v), scale=scale)
        got = out.cpu()[torch.from_numpy(idx).long()].float().numpy()
        err = np.abs(got - ref)
        bound = 2.0**-8 * (vmax + np.abs(ref)) + 1e-3
        assert np.all(err <= bound), (scale, float((err - bound).max()))
        assert err.sum() / np.abs(ref).sum() <= ATT_MEAN_REL


def test_attention_permutation_invariance(J):
    # attention over [fresh active ; frozen] concatenated equals the token-ordered cache
    N, H, d, n_act = 500, 2, 128, 90
    g = np.random.default_rng(8)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.normal_bf16((n_act, H, d), 21)
    k = synth.normal_bf16((N, H, d), 22)
    v = synth.normal_bf16((N, H, d), 23)
    cat = np.concatenate([idx, np.setdiff1d(np.arange(N), idx)])
    out_a = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    out_b = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(idx).cuda(), out_a)
    J.active_attention(dev_bf16(q), dev_bf16(k[cat]), dev_bf16(v[cat]),
                       torch.from_numpy(idx).cuda(), out_b)
    a, b = out_a[idx].float(), out_b[idx].float()
    assert float((a - b).abs().sum() / a.abs().sum()) <= ATT_MEAN_REL


def test_attention_deterministic_and_bad_index(J):
    N, H, d, n_act = 300, 2, 128, 40
    q = synth.normal_bf16((n_act, H, d), 31)
    k = synth.normal_bf16((N, H, d), 32)
    v = synth.normal_bf16((N, H, d), 33)
    idx = np.arange(0, 2 * n_act, 2, dtype=np.int32)
    outs = []
    for _ in range(3):
        o = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
        J.active_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(idx).cuda(), o)
        outs.append(o)
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    bad = idx.copy()
    bad[3] = N
    o = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(bad).cuda(), o)
    assert J.device_error() == 6
    # row 3 is out of range and row 4 (id 8) is not above its predecessor (N):
    # both are skipped, every other row is computed as before
    keep = np.delete(np.arange(n_act), [3, 4])
    assert torch.equal(o[idx[keep]], outs[0][idx[keep]])
    assert torch.count_nonzero(o[idx[[3, 4]]].float()) == 0


# ---------------------------------------------------------------- idx contract
# idx must be strictly ascending (what the schedule emits).  A row whose id is
# not above the previous row's id (a duplicate or a step back) raises
# JANO_EINDEX and is skipped; the other rows are computed as usual.
BAD_IDX = np.array([0, 2, 2, 5, 4, 9, 11, 13], dtype=np.int32)   # rows 2 (dup) and 4 (back)
BAD_ROWS = [2, 4]
GOOD_ROWS = [0, 1, 3, 5, 6, 7]


def test_kv_scatter_rejects_duplicate_and_descending_ids(J):
    N, H, d = 16, 2, 64
    kc = synth.normal_bf16((N, H, d), 41).cuda()
    vc = synth.normal_bf16((N, H, d), 42).cuda()
    before_k, before_v = kc.clone(), vc.clone()
    ka = synth.normal_bf16((BAD_IDX.size, H, d), 43).cuda()
    va = synth.normal_bf16((BAD_IDX.size, H, d), 44).cuda()
    J.kv_scatter(ka, va, torch.from_numpy(BAD_IDX).cuda(), kc, vc)
    assert J.device_error() == 6
    good = BAD_IDX[GOOD_ROWS]
    assert torch.equal(kc[good], ka[GOOD_ROWS]) and torch.equal(vc[good], va[GOOD_ROWS])
    # token 2 holds row 1 (the duplicate row 2 was skipped); token 4 is untouched
    rest = np.setdiff1d(np.arange(N), good)
    assert torch.equal(kc[rest], before_k[rest]) and torch.equal(vc[rest], before_v[rest])


@pytest.mark.parametrize("split", [1, 2])
def test_attention_rejects_duplicate_and_descending_ids(J, split):
    N, H, d = 300, 2, 128
    q = synth.normal_bf16((BAD_IDX.size, H, d), 45)
    k = synth.normal_bf16((N, H, d), 46)
    v = synth.normal_bf16((N, H, d), 47)
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(BAD_IDX).cuda(), out,
                       split=split)
    assert J.device_error() == 6
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v),
                                  rows=np.array(GOOD_ROWS, dtype=np.int32))
    got = out.cpu()[torch.from_numpy(BAD_IDX[GOOD_ROWS]).long()].float().numpy()
    mx, mr = attention_errors(got, ref)
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL
    # token 4 (only named by the skipped row 4) stays unwritten
    assert torch.count_nonzero(out[4].float()) == 0
