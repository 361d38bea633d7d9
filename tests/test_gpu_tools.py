"""The timing modules run end to end on small shapes and print one JSON
line each (they are the commands the profile summaries cite)."""
import json

import pytest
import torch

pytestmark = pytest.mark.gpu


def _lines(capsys):
    out = capsys.readouterr().out.strip().splitlines()
    return [json.loads(l) for l in out if l.startswith("{")]


def test_projection_run(capsys):
    from kv_cache_analyzer_b200 import projection_run
    projection_run.main(["--tokens", "1024", "--hidden", "256", "--active", "300", "--reps", "2"])
    (d,) = _lines(capsys)
    assert d["qkv_project"]["TFLOP/s"] > 0 and d["out_proj_scatter"]["TFLOP/s"] > 0


def test_spectral_run(capsys):
    from kv_cache_analyzer_b200 import spectral_run
    spectral_run.main(["--channels", "4", "--frames", "3", "--height", "18", "--width", "40", "--reps", "2"])
    (d,) = _lines(capsys)
    assert d["shape"]["n_blocks"] == 3 * 5 * 10
    assert d["fft_score"]["GB/s"] > 0 and d["block_scores"]["GB/s"] > 0 and d["plain_read"]["GB/s"] > 0


def test_sharding_run(capsys):
    from kv_cache_analyzer_b200 import sharding_run
    sharding_run.main(["--ranks", "1", "2", "3", "--frames", "3", "--height", "16", "--width", "32",
                       "--heads", "6", "--reps", "2"])
    lines = _lines(capsys)
    assert [d["ranks"] for d in lines] == [1, 2, 3]
    for d in lines:
        assert sum(p["heads"] for p in d["per_rank"]) == 6
        assert sum(p["frames"] for p in d["per_rank"]) == 3
        assert d["n_active"] == lines[0]["n_active"] > 0
    torch.cuda.synchronize()


def test_split_run(capsys):
    from kv_cache_analyzer_b200 import split_run
    split_run.main(["--case", "2048", "2", "300", "--case", "300", "1", "40", "--splits", "1", "2", "3", "5",
                    "--reps", "2"])
    lines = _lines(capsys)
    assert [d["n_act"] for d in lines] == [300, 40]
    assert set(lines[0]["TFLOP/s"]) == {"1", "2", "3", "5"} and lines[0]["chosen"] >= 1
    assert set(lines[1]["TFLOP/s"]) == {"1", "2", "3"}     # 3 key tiles: at most 3 ranges
    assert lines[1]["chosen"] == 1                          # under 8 key tiles per range: no split
    assert all(v > 0 for d in lines for v in d["TFLOP/s"].values())
