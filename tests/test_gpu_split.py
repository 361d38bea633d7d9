"""Key-split attention (jano_active_attention_split) against the fp64 oracle.

The keys of every query tile are cut into n_split ranges of whole 128-key
tiles, one CTA each; a merge pass rescales each range's unnormalised output
and sum by 2^(m_s - max m) and divides.  Same tolerances as the unsplit
kernel: max-abs 2e-2 and mean-rel 5e-3 of the fp64 values.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from workloads import attention_errors, cta_position_rows, oracle_attention_rows, sample_rows

pytestmark = pytest.mark.gpu

ATT_MAX_ABS = 2e-2
ATT_MEAN_REL = 5e-3


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


def _case(N, n_act, H, d, seed):
    g = np.random.default_rng(seed)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.normal_bf16((n_act, H, d), seed + 1)
    k = synth.normal_bf16((N, H, d), seed + 2)
    v = synth.normal_bf16((N, H, d), seed + 3)
    return idx, q, k, v


def _run(J, q, k, v, idx, split, scale=None):
    N, H, d = k.shape
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    J.active_attention(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(), out,
                       scale=scale, split=split)
    return out


@pytest.mark.parametrize("N,n_act,H,d,split", [
    (1000, 300, 3, 128, 2),      # 8 key tiles, 4 per CTA
    (1000, 300, 3, 64, 3),       # uneven ranges (3/3/2 tiles), d = 64
    (2049, 129, 2, 128, 5),      # last key tile holds one key
    (640, 50, 1, 128, 5),        # as many splits as key tiles
    (300, 40, 2, 128, 3),        # one ragged tile in the last range
    (4096, 600, 2, 128, 7),
])
def test_split_matches_oracle(J, N, n_act, H, d, split):
    idx, q, k, v = _case(N, n_act, H, d, N * 3 + split)
    out = _run(J, q, k, v, idx, split)
    assert J.device_error() == 0
    got = out.cpu()
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v))
    mx, mr = attention_errors(got[torch.from_numpy(idx).long()].float().numpy(), ref)
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL, (mx, mr)
    # only the rows of idx are written
    mask = torch.ones(N, dtype=torch.bool)
    mask[torch.from_numpy(idx).long()] = False
    assert torch.count_nonzero(got[mask].float()) == 0


def test_split_agrees_with_unsplit_and_is_deterministic(J):
    idx, q, k, v = _case(3000, 500, 2, 128, 77)
    one = _run(J, q, k, v, idx, 1)
    outs = [_run(J, q, k, v, idx, 4) for _ in range(3)]
    assert J.device_error() == 0
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    a, b = one[idx].float(), outs[0][idx].float()
    # both round P and the output to BF16; the ranges only change which
    # running maximum each key's P is taken against, so the two agree within
    # the attention tolerance
    assert float((a - b).abs().max()) <= ATT_MAX_ABS
    assert float((a - b).abs().sum() / a.abs().sum()) <= ATT_MEAN_REL


def test_split_peaked_softmax(J):
    # logits spread over many binades: each range's running max differs, the
    # merge rescales by 2^(m_s - M) with |m_s - M| large
    N, H, d, n_act = 1500, 2, 64, 130
    g = np.random.default_rng(15)
    idx = np.sort(g.choice(N, size=n_act, replace=False)).astype(np.int32)
    q = synth.tensor_of(synth.bf16_bits((3.0 * g.standard_normal((n_act, H, d))).astype(np.float32)))
    base = 3.0 * g.standard_normal((N, H, d)) * np.linspace(0.2, 2.0, N)[:, None, None]
    k = synth.tensor_of(synth.bf16_bits(base.astype(np.float32)))
    v = synth.normal_bf16((N, H, d), 19)
    vmax = float(v.float().abs().amax())
    out = _run(J, q, k, v, idx, 4)
    assert J.device_error() == 0
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v))
    got = out.cpu()[torch.from_numpy(idx).long()].float().numpy()
    err = np.abs(got - ref)
    # P rounded to BF16 moves o by at most 2^-8 max|v|, the BF16 output by 2^-8 |o|
    bound = 2.0**-8 * (vmax + np.abs(ref)) + 1e-3
    assert np.all(err <= bound), float((err - bound).max())
    assert err.sum() / np.abs(ref).sum() <= ATT_MEAN_REL


def test_split_bad_index_raises_and_skips_the_row(J):
    idx, q, k, v = _case(600, 40, 2, 128, 5)
    good = _run(J, q, k, v, idx, 3)
    assert J.device_error() == 0
    bad = idx.copy()
    bad[7] = 600
    out = _run(J, q, k, v, bad, 3)
    assert J.device_error() == 6
    # row 7 is out of range and row 8 is not above its predecessor (600): both skipped
    keep = np.delete(np.arange(idx.size), [7, 8])
    assert torch.equal(out[idx[keep]], good[idx[keep]])


def test_caller_workspace_is_reused(J):
    idx, q, k, v = _case(1200, 200, 2, 128, 9)
    ws_bytes = J.jano_active_attention_workspace_bytes(200, 2, 128, 3)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    N, H, d = k.shape
    a = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    for out in (a, b):
        J.active_attention(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(), out,
                           split=3, workspace=ws)
    assert J.device_error() == 0
    assert torch.equal(a, b)


def test_small_due_set_of_the_sweep_takes_a_split(J):
    # the 10% point of the active-fraction sweep: 3,276 of 32,760 tokens,
    # 12 heads, d = 128 -- 13 query-tile pairs x 12 heads = 156 CTAs
    N, H, d, n_act = 32760, 12, 128, 3276
    split = J.jano_active_attention_splits(n_act, N, H, d)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if sms >= 100:
        assert split > 1
    idx, q, k, v = _case(N, n_act, H, d, 123)
    out = _run(J, q, k, v, idx, None)
    assert J.device_error() == 0
    rows = sample_rows(n_act, 4, seed=3)
    ref = oracle.active_attention(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v), rows=rows)
    got = out.cpu()[torch.from_numpy(idx[rows]).long()].float().numpy()
    mx, mr = attention_errors(got, ref)
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL, (mx, mr)


@pytest.mark.parametrize("frac", [0.25, 0.5, 0.75, 1.0])
def test_sweep_points_match_oracle(J, frac):
    # the other points of the active-fraction sweep on the 32,760-token,
    # 12-head shape: the top `frac` of the smooth per-token field is due (the
    # sweep's first interleaved step), attention over the whole cache with the
    # library's split choice for that due set (the 50% point splits keys)
    w = synth.WORKLOADS["schedule50"]
    N, H, d = w.n_tokens, w.heads, w.d
    TF, TH, TW = w.grid
    field = synth.token_field(TF, TH, TW, seed=w.seed * 10 + 1, sigma=w.field_sigma)
    lv = oracle.classify(field, frac, 1.0 - frac)
    idx = np.flatnonzero(lv == 3).astype(np.int32)
    n_act = idx.size
    assert n_act == int(round(frac * 10000)) * N // 10000
    q = synth.normal_bf16((n_act, H, d), 700 + int(frac * 100))
    k = synth.normal_bf16((N, H, d), 801)
    v = synth.normal_bf16((N, H, d), 802)
    split = J.jano_active_attention_splits(n_act, N, H, d)
    out = _run(J, q, k, v, idx, None)
    assert J.device_error() == 0
    rows = cta_position_rows(n_act, n_ctas=16, seed=int(frac * 100))
    ref = oracle_attention_rows(synth.bits_of(q), synth.bits_of(k), synth.bits_of(v), rows)
    got = out.cpu()[torch.from_numpy(idx[rows]).long()].float().numpy()
    mx, mr = attention_errors(got, ref)
    print(f"sweep {frac:.2f}: n_act {n_act}, split {split}, rows {rows.size}, max-abs {mx:.2e}, mean-rel {mr:.2e}")
    assert mx <= ATT_MAX_ABS and mr <= ATT_MEAN_REL, (mx, mr)
