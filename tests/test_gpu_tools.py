"""The measurement modes of bench.py run end to end on small shapes and print
one JSON line each (they are the commands the profile summaries cite)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*argv, timeout=900):
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv],
                       capture_output=True, text=True, timeout=timeout, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]


def test_projection_mode():
    (d,) = _bench("--mode", "projection", "--tokens", "1024", "--hidden", "256", "--active", "300",
                  "--reps", "2")
    assert d["qkv_project"]["TFLOP/s"] > 0 and d["out_proj_scatter"]["TFLOP/s"] > 0


def test_spectral_mode():
    (d,) = _bench("--mode", "spectral", "--channels", "4", "--frames", "3", "--height", "18",
                  "--width", "40", "--reps", "2")
    assert d["shape"]["n_blocks"] == 3 * 5 * 10
    assert d["fft_score"]["GB/s"] > 0 and d["block_scores"]["GB/s"] > 0 and d["plain_read"]["GB/s"] > 0


def test_sharded_mode():
    lines = _bench("--mode", "sharded", "--ranks", "1", "2", "3", "--frames", "3", "--height", "16",
                   "--width", "32", "--heads", "6", "--reps", "2")
    assert [d["ranks"] for d in lines] == [1, 2, 3]
    for d in lines:
        assert sum(p["heads"] for p in d["per_rank"]) == 6
        assert sum(p["frames"] for p in d["per_rank"]) == 3
        assert d["n_active"] == lines[0]["n_active"] > 0


def test_splits_mode():
    lines = _bench("--mode", "splits", "--case", "2048", "2", "300", "--case", "300", "1", "40",
                   "--splits", "1", "2", "3", "5", "--reps", "2")
    assert [d["n_act"] for d in lines] == [300, 40]
    assert set(lines[0]["TFLOP/s"]) == {"1", "2", "3", "5"} and lines[0]["chosen"] >= 1
    assert set(lines[1]["TFLOP/s"]) == {"1", "2", "3"}     # 3 key tiles: at most 3 ranges
    assert lines[1]["chosen"] == 1                          # under 8 key tiles per range: no split
    assert all(v > 0 for d in lines for v in d["TFLOP/s"].values())


def test_schedule50_mode():
    (d,) = _bench("--workload", "schedule50", "--reps", "1", "--fractions", "0.1,1.0")
    assert d["mode"] == "schedule50" and d["due_token_steps"] > 0
    assert 1.0 < d["speedup_vs_full"] and [p["fraction"] for p in d["sweep"]] == [0.1, 1.0]
