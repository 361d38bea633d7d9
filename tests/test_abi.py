"""The C-ABI library loads and exports every symbol include/jano.h declares,
and host-side argument validation rejects bad calls without touching a GPU."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "jano.h")).read()
    return re.findall(r"JANO_API\s+[\w\s\*]+?\b(jano_\w+)\s*\(", txt)


@pytest.fixture(scope="module")
def jl():
    from kv_cache_analyzer_b200 import build
    build.build()
    import kv_cache_analyzer_b200 as j
    return j


def test_header_declares_the_boundary():
    names = set(_declared())
    for fn in ("jano_block_scores", "jano_classify", "jano_build_schedule",
               "jano_kv_scatter", "jano_active_attention"):
        assert fn in names


def test_library_exports_every_declared_symbol(jl):
    L = jl.lib()
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) == set(jl.EXPORTS)


def test_status_strings_and_version(jl):
    assert jl.jano_version() >= 100
    assert jl.jano_status_str(0) == "ok"
    assert "index" in jl.jano_status_str(6)


def test_workspace_query_is_host_only(jl):
    g = jl.Geometry(21, 90, 160, (1, 4, 4), (1, 2, 2))
    n = jl.jano_build_schedule_workspace_bytes(g.c())
    # token levels (75600 B) + one int32 [3][74] table, 16-byte rounded
    assert n == 75600 + 896
    bad = jl.Geometry(21, 91, 160, (1, 4, 4), (1, 2, 2))     # H not divisible by ph
    assert jl.jano_build_schedule_workspace_bytes(bad.c()) == 0


def test_host_validation_rejects_before_any_launch(jl):
    L = jl.lib()
    nil = C.c_void_p(0)
    fake = C.c_void_p(256)          # never dereferenced: validation fails first
    # d not in {64, 128}
    assert L.jano_active_attention(fake, fake, fake, fake, 10, 100, 2, 96, 0.1, fake, nil) == 4
    # non-positive scale
    assert L.jano_active_attention(fake, fake, fake, fake, 10, 100, 2, 128, 0.0, fake, nil) == 1
    # misaligned pointer
    assert L.jano_active_attention(C.c_void_p(258), fake, fake, fake, 10, 100, 2, 128, 0.1, fake, nil) == 3
    # n_act == 0 is a no-op that succeeds without a device
    assert L.jano_active_attention(nil, nil, nil, nil, 0, 100, 2, 128, 0.1, nil, nil) == 0
    assert L.jano_kv_scatter(nil, nil, nil, 0, 2, 128, nil, nil, 100, nil) == 0
    assert L.jano_kv_scatter(fake, fake, fake, -1, 2, 128, fake, fake, 100, nil) == 1
    # row of heads*d BF16 not a multiple of 16 bytes
    assert L.jano_kv_scatter(fake, fake, fake, 3, 1, 4, fake, fake, 100, nil) == 4
    # classify fractions out of range / summing above 1
    assert L.jano_classify(fake, 10, 0.7, 0.7, fake, nil) == 1
    assert L.jano_classify(fake, 10, -0.1, 0.2, fake, nil) == 1
    assert L.jano_classify(fake, 0, 0.1, 0.2, fake, nil) == 1
    # block scores: K < 2, W not a multiple of 4
    g = jl.Geometry(4, 32, 32).c()
    assert L.jano_block_scores(fake, 1, 16, C.byref(g), 0.5, 0.5, fake, nil) == 1
    g2 = jl.Geometry(4, 32, 30, (1, 4, 4), (1, 2, 2)).c()
    assert L.jano_block_scores(fake, 5, 16, C.byref(g2), 0.5, 0.5, fake, nil) == 4
    # schedule: warm-up + cool-down longer than T, index capacity too small
    g3 = jl.Geometry(4, 32, 32).c()
    bad = jl.Schedule(T=4, warmup=3, cooldown=2).c()
    assert L.jano_build_schedule(fake, C.byref(g3), C.byref(bad), fake, fake, 10**6, nil, fake,
                                 10**6, nil) == 1
    ok = jl.Schedule(T=4, warmup=1, cooldown=1).c()
    assert L.jano_build_schedule(fake, C.byref(g3), C.byref(ok), fake, fake, 10, nil, fake,
                                 10**6, nil) == 1
    # projections: k or n not a multiple of 8, misaligned operand, m beyond
    # the rows without a gather, an empty call, hd not a multiple of 128
    assert L.jano_gather_gemm(fake, 64, nil, 16, fake, 60, 64, nil, fake, 64, nil) == 4
    assert L.jano_gather_gemm(fake, 64, nil, 16, fake, 64, 60, nil, fake, 64, nil) == 4
    assert L.jano_gather_gemm(C.c_void_p(264), 64, nil, 16, fake, 64, 64, nil, fake, 64, nil) == 3
    assert L.jano_gather_gemm(fake, 8, nil, 16, fake, 64, 64, nil, fake, 64, nil) == 2
    assert L.jano_gather_gemm(nil, 8, nil, 0, nil, 64, 64, nil, nil, 64, nil) == 0
    assert L.jano_qkv_project(fake, 100, fake, 10, fake, 96, 64, fake, fake, fake, nil) == 4
    assert L.jano_qkv_project(nil, 100, nil, 0, nil, 128, 64, nil, nil, nil, nil) == 0
    # FFT score: negative cutoff, no channels, NULL snapshot, a block of more
    # than 256 elements
    g4 = jl.Geometry(4, 32, 32, (1, 4, 4), (1, 2, 2)).c()
    assert L.jano_fft_scores(fake, 16, C.byref(g4), -1, fake, nil) == 1
    assert L.jano_fft_scores(fake, 0, C.byref(g4), 1, fake, nil) == 1
    assert L.jano_fft_scores(nil, 16, C.byref(g4), 1, fake, nil) == 1
    g5 = jl.Geometry(4, 32, 32, (4, 8, 16), (1, 2, 2)).c()
    assert L.jano_fft_scores(fake, 16, C.byref(g5), 1, fake, nil) == 4
    # key-split attention: split count out of range (0; more splits than
    # key tiles of 128), NULL / short / misaligned workspace, an empty call
    need = L.jano_active_attention_workspace_bytes(300, 4, 128, 3)
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 128, 0.1, 0, fake,
                                         need, fake, nil) == 1
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 128, 0.1, 9, fake,
                                         10**9, fake, nil) == 1
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 128, 0.1, 3, nil,
                                         need, fake, nil) == 1
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 128, 0.1, 3, fake,
                                         need - 1, fake, nil) == 1
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 128, 0.1, 3,
                                         C.c_void_p(264), need, fake, nil) == 3
    assert L.jano_active_attention_split(nil, nil, nil, nil, 0, 1024, 4, 128, 0.1, 3, nil, 0,
                                         nil, nil) == 0
    assert L.jano_active_attention_split(fake, fake, fake, fake, 300, 1024, 4, 96, 0.1, 3, fake,
                                         need, fake, nil) == 4


def test_split_attention_workspace_and_choice_are_host_only(jl):
    # n_split rows of fp32 partials (256-byte rounded), then (m, l) pairs
    assert jl.jano_active_attention_workspace_bytes(300, 4, 128, 3) == 3 * 300 * 4 * 128 * 4 + 3 * 300 * 4 * 8
    assert jl.jano_active_attention_workspace_bytes(5, 3, 64, 2) == 7680 + 2 * 5 * 3 * 8
    assert jl.jano_active_attention_workspace_bytes(300, 4, 128, 1) == 0
    assert jl.jano_active_attention_workspace_bytes(0, 4, 128, 3) == 0
    # without a device the library recommends no split
    if not __import__("torch").cuda.is_available():
        assert jl.jano_active_attention_splits(3276, 32760, 12, 128) == 1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch, jl):
    monkeypatch.setattr(jl, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(jl, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        jl.lib()


def test_every_workload_geometry_passes_host_support_checks(jl):
    # On a machine without a GPU a supported call gets past validation and
    # fails only at the device lookup (JANO_ECUDA); an unsupported shape
    # would return JANO_EUNSUPPORTED (4) before that.
    import synth
    L = jl.lib()
    fake = C.c_void_p(256)
    for name, w in synth.WORKLOADS.items():
        g = jl.Geometry(w.F, w.H, w.W, w.block, w.patch).c()
        code = L.jano_block_scores(fake, w.K, w.C, C.byref(g), 0.5, 0.5, fake, None)
        assert code != 4, name
    for shape, block in [((3, 2, 3, 9, 12), (1, 4, 4)), ((4, 3, 5, 6, 8), (2, 3, 2)),
                         ((6, 1, 1, 16, 16), (1, 2, 2)), ((3, 1, 2, 4, 20), (1, 4, 8)),
                         ((9, 64, 8, 64, 256), (2, 8, 8)), ((6, 16, 1, 720, 1280), (1, 4, 4))]:
        K1, Cc, F, H, W = shape
        g = jl.Geometry(F, H, W, block, (1, 1, 1)).c()
        assert L.jano_block_scores(fake, K1 - 1, Cc, C.byref(g), 0.5, 0.5, fake, None) != 4, shape


def test_split_choice_on_a_given_sm_count(jl):
    f = jl.jano_active_attention_splits_on
    # the shapes of the measured split sweep, 148 SMs (B200)
    assert [f(n, 32760, 12, 128, 148) for n in (1638, 3276, 8190, 16380, 24570, 32760)] == [3, 4, 1, 2, 1, 1]
    assert f(18900, 75600, 5, 128, 148) == 2        # a rank of the 8-way head-sharded step
    assert f(18900, 75600, 40, 128, 148) == 1       # the large step's due sets never split
    assert f(41580, 75600, 40, 128, 148) == 1
    assert f(75600, 75600, 40, 128, 148) == 1
    # fewer than 16 key tiles: no range of 8+ tiles to split into
    assert f(100, 1000, 1, 128, 148) == 1
    assert f(1, 2049, 1, 64, 148) == 2              # 17 tiles: two ranges of 8+
    # invalid arguments
    assert f(100, 32760, 12, 96, 148) == 1
    assert f(100, 32760, 12, 128, 0) == 1
    assert f(0, 32760, 12, 128, 148) == 1
    for sms in (1, 16, 148, 1000):
        for n in (1, 300, 3276, 40000):
            for N in (128, 1024, 32760, 75600):
                z = f(n, N, 4, 128, sms)
                assert 1 <= z <= 16 and (z == 1 or ((N + 127) // 128) // z >= 8)


def test_noalloc_limit_is_exactly_its_scratch(jl):
    # The static scratch is 1 MiB: align16(n) + align16(12 * ceil(n / 1024))
    # bytes for n tokens.  2699 x 384 = 1,036,416 tokens need exactly 1 MiB;
    # one token more (a 1 x 1,036,417 row) needs 1,048,592 bytes.
    L = jl.lib()
    at = jl.Geometry(1, 2699, 384, (1, 1, 1), (1, 1, 1))
    over = jl.Geometry(1, 1, 1_036_417, (1, 1, 1), (1, 1, 1))
    assert at.n_tokens == 1_036_416 and over.n_tokens == 1_036_417
    assert jl.jano_build_schedule_workspace_bytes(at.c()) == 1 << 20
    assert jl.jano_build_schedule_workspace_bytes(over.c()) == (1 << 20) + 16
    c = jl.Schedule(2, 1, 1, 1, 1).c()
    nil = C.c_void_p(0)
    g_over = over.c()
    # one token over the limit: rejected before any CUDA call (no device needed)
    assert L.jano_build_schedule_noalloc(nil, C.byref(g_over), C.byref(c), nil, nil, 10**9, nil,
                                         nil) == 4
    # at the limit the size check passes; the call then fails later for other
    # reasons (no device here -> JANO_ECUDA, NULL buffers -> JANO_EINVAL), never
    # with JANO_EUNSUPPORTED
    g_at = at.c()
    assert L.jano_build_schedule_noalloc(nil, C.byref(g_at), C.byref(c), nil, nil, 10**9, nil,
                                         nil) in (1, 8)
