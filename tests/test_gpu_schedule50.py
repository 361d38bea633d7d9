"""The full 50-step interleaved schedule at 32,760 tokens, 12 heads, d=128,
with the KV cache carried across steps, against the fp64 oracle.

Chain: block scores of the latent history (blocks = token patches) ->
classify 30/30/40 -> 50-step schedule (5 warm-up, Moderate every 2, Static
every 4, 5 cool-down) -> per step: scatter the fresh K/V of the due tokens,
attend with their queries.  The oracle replays every scatter on the host;
caches are compared bit for bit and attention on sampled rows at steps of
every kind (warm-up, Active only, Active+Moderate, all levels, cool-down):
about a hundred rows per sampled step, one in each query tile and TMEM lane
quarter of a spread of CTAs plus the first and last rows, all heads.
Resuming from the state saved after step 25 reproduces the final output and
caches bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from workloads import attention_errors, cta_position_rows, oracle_attention_rows

pytestmark = pytest.mark.gpu

# warm-up (0), Active only (5), Active + Moderate (6), all levels (8, 44),
# an Active + Moderate step mid-way (25), the first and last cool-down steps (45, 49)
SAMPLED_STEPS = (0, 5, 6, 8, 25, 44, 45, 49)


@pytest.fixture(scope="module")
def J():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    j.lib()
    return j


def test_fifty_steps_with_carried_cache_and_resume(J):
    w = synth.WORKLOADS["schedule50"]
    N, H, d = w.n_tokens, w.heads, w.d
    dev = torch.device("cuda")
    # ---- a1..a3 on the GPU, checked stage-wise against the oracle
    lat = synth.latent_history(w.K, w.C, w.F, w.H, w.W, seed=w.seed)
    geom = J.Geometry(w.F, w.H, w.W, w.block, w.patch)
    scores = J.block_scores(torch.from_numpy(lat).to(dev), geom)
    s_host = scores.cpu().numpy()
    ref_s = oracle.block_scores(lat, w.block)
    assert np.all(np.abs(s_host - ref_s) <= 1e-5 * np.abs(ref_s) + 1e-7)
    levels = J.classify(scores, w.frac_active, w.frac_static)
    lv_host = levels.cpu().numpy()
    np.testing.assert_array_equal(lv_host, oracle.classify(s_host, w.frac_active, w.frac_static))
    sched = J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static)
    off, idx, _ = J.build_schedule(levels, geom, sched)
    off_h = off.cpu().numpy()
    idx_h = idx.cpu().numpy()[: off_h[-1]]
    r_off, r_idx, _ = oracle.build_schedule(lv_host, (w.F, w.H, w.W), w.block, w.patch, w.T, w.warmup,
                                            w.cooldown, w.period_moderate, w.period_static)
    np.testing.assert_array_equal(off_h, r_off)
    np.testing.assert_array_equal(idx_h, r_idx)
    assert off_h[-1] == 10 * N + 40 * (lv_host == 3).sum() + 20 * (lv_host == 2).sum() + 10 * (lv_host == 1).sum()

    # ---- seeded pools and the initial cache
    base = 5000
    pq, pk, pv = (synth.normal_bf16((N, H, d), base + i) for i in range(3))
    kc0, vc0 = synth.normal_bf16((N, H, d), base + 3), synth.normal_bf16((N, H, d), base + 4)
    kc, vc = kc0.to(dev), vc0.to(dev)
    out = torch.zeros(N, H, d, dtype=torch.bfloat16, device=dev)
    okc, ovc = synth.bits_of(kc0).copy(), synth.bits_of(vc0).copy()

    def step_inputs(s):
        toks = idx_h[off_h[s]:off_h[s + 1]]
        rows = torch.from_numpy(synth.step_rows(toks, s, N))
        return toks, pq[rows].contiguous(), pk[rows].contiguous(), pv[rows].contiguous()

    def gpu_step(s):
        toks, q, k, v = step_inputs(s)
        t_dev = idx[off_h[s]:off_h[s + 1]]
        J.kv_scatter(k.to(dev), v.to(dev), t_dev, kc, vc)
        J.active_attention(q.to(dev), kc, vc, t_dev, out)
        return toks, q, k, v

    saved = None
    for s in range(w.T):
        if s == 25:
            saved = (kc.clone(), vc.clone(), out.clone())
        toks, q, k, v = gpu_step(s)
        okc, ovc = oracle.kv_scatter(synth.bits_of(k), synth.bits_of(v), toks, okc, ovc)
        if s in SAMPLED_STEPS:
            assert J.device_error() == 0
            np.testing.assert_array_equal(synth.bits_of(kc.cpu()), okc)
            np.testing.assert_array_equal(synth.bits_of(vc.cpu()), ovc)
            rows = cta_position_rows(toks.size, n_ctas=12, seed=s)
            ref = oracle_attention_rows(synth.bits_of(q), okc, ovc, rows)
            got = out[torch.from_numpy(toks[rows]).long().to(dev)].float().cpu().numpy()
            mx, mr = attention_errors(got, ref)
            print(f"step {s}: {toks.size} due tokens, rows {rows.size}, max-abs {mx:.2e}, mean-rel {mr:.2e}")
            assert mx <= 2e-2 and mr <= 5e-3
    final = (kc.clone(), vc.clone(), out.clone())
    # ---- resume from the state saved after step 25
    kc.copy_(saved[0]); vc.copy_(saved[1]); out.copy_(saved[2])
    for s in range(25, w.T):
        gpu_step(s)
    assert J.device_error() == 0
    for a, b in zip(final, (kc, vc, out)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
