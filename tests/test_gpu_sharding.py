"""The step sharded over ranks (frame slabs for the analyzer, head ranges for
scatter and attention), emulated on one GPU: the ranks' kernels run one
after another, each on its own buffers, and the all-gather of block scores
is a concatenation.  No rank waits on another inside a kernel, so running
them in sequence is exact emulation.

Two checks: every rank's scores, schedule, cache heads and output heads
equal the unsharded step's (bit for bit where both take the same key split);
and every rank's results match the fp64 oracle on the rank's own share --
its slab's block scores, the gathered scores, levels and schedule, its cache
heads after the scatter (bit for bit) and sampled attention rows of its
heads (max-abs 2e-2, mean-rel 5e-3)."""
import os
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _geoms(J, w):
    return (J.Geometry(w.F, w.H, w.W, w.block, w.patch), J.Geometry(w.F, w.H, w.W, w.patch, w.patch),
            J.Schedule(w.T, w.warmup, w.cooldown, w.period_moderate, w.period_static))


def _bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu()


def _run_shards(J, w, world, inp, k_cache, v_cache, n_cap, stream, step):
    """Every rank's share of one step, run one rank after another on this GPU;
    the all-gather of block scores is a concatenation."""
    from kv_cache_analyzer_b200.sharding import ShardedHotPath
    lg, tg, sc = _geoms(J, w)
    shards = []
    for r in range(world):
        sh = ShardedHotPath(rank=r, world=world, K=w.K, C=w.C, latent_geom=lg, token_geom=tg,
                            heads=w.heads, d=w.d, frac_active=w.frac_active,
                            frac_static=w.frac_static, sched=sc, stream=stream)
        sh.set_activations(n_cap)
        sh.load_latent(inp["lat"])
        with torch.cuda.stream(stream):
            sh.field.copy_(inp["field"])
            for k in ("q_act", "k_act", "v_act"):
                getattr(sh, k).copy_(sh.head_slice(inp[k]))
            sh.k_cache.copy_(sh.head_slice(k_cache)); sh.v_cache.copy_(sh.head_slice(v_cache))
        shards.append(sh)
    assert sum(sh.heads for sh in shards) == w.heads
    assert sum(sh.counts[sh.rank] for sh in shards) == lg.n_blocks
    # a1 on every rank, then the gather, then a2..a5 on every rank
    for sh in shards:
        sh.run_local_scores()
    with torch.cuda.stream(stream):
        full = torch.cat([sh.local_scores() for sh in shards])
        for sh in shards:
            sh.scores.copy_(full)
    for sh in shards:
        sh.run_after_gather()
    stream.synchronize()
    for sh in shards:
        sh.host_offsets = sh.offsets.cpu().tolist()
        sh.run_head_kernels(step)
    stream.synchronize()
    assert J.device_error() == 0
    return shards


@pytest.mark.parametrize("name,world", [("tiny", 2), ("small", 2), ("small", 3), ("large", 8),
                                        ("small", 5), ("image", 3), ("tiny", 8)])
def test_sharded_step_equals_unsharded(name, world):
    # uneven shares (12 heads and 21 frames over 5 ranks), ranks without a
    # frame-block (one frame over 3 ranks) and ranks without a head or a
    # frame-block (4 heads and 4 frames over 8 ranks) included
    import bench
    import synth
    import kv_cache_analyzer_b200 as J
    from kv_cache_analyzer_b200.pipeline import HotPath
    w = synth.WORKLOADS[name]
    inp, k_cache, v_cache, n_cap = bench.make_inputs(w)
    lg, tg, sc = _geoms(J, w)
    stream = torch.cuda.Stream()
    step = w.warmup

    ref = HotPath(K=w.K, C=w.C, latent_geom=lg, token_geom=tg, heads=w.heads, d=w.d,
                  frac_active=w.frac_active, frac_static=w.frac_static, sched=sc, stream=stream)
    ref.set_activations(n_cap)
    with torch.cuda.stream(stream):
        ref.lat.copy_(inp["lat"]); ref.field.copy_(inp["field"])
        ref.q_act.copy_(inp["q_act"]); ref.k_act.copy_(inp["k_act"]); ref.v_act.copy_(inp["v_act"])
        ref.k_cache.copy_(k_cache); ref.v_cache.copy_(v_cache)
    stream.synchronize()
    ref.plan()
    ref.run_step_kernels(step)
    stream.synchronize()
    assert J.device_error() == 0

    shards = _run_shards(J, w, world, inp, k_cache, v_cache, n_cap, stream, step)

    s_ref = _bits(ref.scores)
    off_ref = ref.offsets.cpu()
    n_due = int(off_ref[-1])
    idx_ref = ref.idx[:n_due].cpu()
    for sh in shards:
        assert torch.equal(_bits(sh.scores), s_ref), f"rank {sh.rank} scores"
        assert torch.equal(sh.offsets.cpu(), off_ref)
        assert torch.equal(sh.idx[:n_due].cpu(), idx_ref)
        for mine, theirs in ((sh.k_cache, ref.k_cache), (sh.v_cache, ref.v_cache)):
            assert torch.equal(_bits(mine), _bits(sh.head_slice(theirs))), f"rank {sh.rank} heads"
        if sh.heads == 0:
            continue
        if sh.last_split == ref.last_split:
            assert torch.equal(_bits(sh.out), _bits(sh.head_slice(ref.out))), f"rank {sh.rank} out"
        else:
            # a rank with fewer heads has fewer CTAs and may split the keys where
            # the whole step did not: the same attention up to the rounding of P
            # and of the output to BF16, so the two agree within the attention
            # tolerance (max-abs 2e-2, mean-rel 5e-3)
            a = sh.head_slice(ref.out).float()
            b = sh.out.float()
            assert float((a - b).abs().max()) <= 2e-2, f"rank {sh.rank} out"
            assert float((a - b).abs().sum() / a.abs().sum()) <= 5e-3, f"rank {sh.rank} out"


@pytest.mark.parametrize("name,world", [("small", 3), ("large", 8)])
def test_sharded_ranks_match_oracle(name, world):
    import bench
    import oracle
    import synth
    import kv_cache_analyzer_b200 as J
    from workloads import attention_errors, cta_position_rows, oracle_attention_rows
    w = synth.WORKLOADS[name]
    inp, k_cache, v_cache, n_cap = bench.make_inputs(w)
    stream = torch.cuda.Stream()
    step = w.warmup
    shards = _run_shards(J, w, world, inp, k_cache, v_cache, n_cap, stream, step)

    lat = inp["lat"].numpy()
    ref_scores = oracle.block_scores(lat, w.block)
    lv = oracle.classify(inp["field"].numpy(), w.frac_active, w.frac_static)
    r_off, r_idx, _ = oracle.build_schedule(lv, (w.F, w.H, w.W), w.patch, w.patch, w.T, w.warmup,
                                            w.cooldown, w.period_moderate, w.period_static)
    sel = r_idx[r_off[step]:r_off[step + 1]]
    n_act = sel.size
    for sh in shards:
        # a1: the rank's own blocks, scored on its slab (with the halo frame)
        if sh.n_local:
            slab = np.ascontiguousarray(lat[:, :, sh.f0:sh.f0 + sh.f_slab])
            ref_local = oracle.block_scores(slab, w.block)[:sh.n_local]
            got_local = sh.local_scores().cpu().numpy()
            assert np.all(np.abs(got_local - ref_local) <= 1e-5 * np.abs(ref_local) + 1e-7), sh.rank
        # after the gather: every block's score, the level split and the schedule
        got = sh.scores.cpu().numpy()
        assert np.all(np.abs(got - ref_scores) <= 1e-5 * np.abs(ref_scores) + 1e-7), sh.rank
        np.testing.assert_array_equal(sh.offsets.cpu().numpy(), r_off)
        np.testing.assert_array_equal(sh.idx[:r_off[-1]].cpu().numpy(), r_idx)
        if sh.heads == 0:
            continue
        # a4: the rank's cache heads, bit for bit
        hs = slice(sh.h_lo, sh.h_hi)
        rk, rv = oracle.kv_scatter(synth.bits_of(inp["k_act"][:n_act, hs]),
                                   synth.bits_of(inp["v_act"][:n_act, hs]), sel,
                                   synth.bits_of(k_cache[:, hs]), synth.bits_of(v_cache[:, hs]))
        np.testing.assert_array_equal(synth.bits_of(sh.k_cache.cpu()), rk)
        np.testing.assert_array_equal(synth.bits_of(sh.v_cache.cpu()), rv)
        # a5: sampled rows of the rank's heads, every grid position reached
        rows = cta_position_rows(n_act, n_ctas=16, seed=sh.rank)
        ref = oracle_attention_rows(synth.bits_of(inp["q_act"][:n_act, hs]), rk, rv, rows)
        got_o = sh.out.cpu()[torch.from_numpy(sel[rows]).long()].float().numpy()
        mx, mr = attention_errors(got_o, ref)
        print(f"{name} rank {sh.rank}/{world}: heads {sh.h_lo}..{sh.h_hi}, split {sh.last_split}, "
              f"rows {rows.size}, max-abs {mx:.2e}, mean-rel {mr:.2e}")
        assert mx <= 2e-2 and mr <= 5e-3, sh.rank
