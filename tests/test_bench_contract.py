"""The benchmark's reference arm (the fp64 oracle on the host cores) prints
one JSON line with the keys the driver reads; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == bench.host_cores()
    assert d["config"]["workload"].startswith("tiny")
    # the same config dict as the GPU arm's, and the timed sample is what ms_per_step reports
    assert d["config"] == bench.workload_config(synth.WORKLOADS["tiny"], 1)
    assert d["extrapolated"] is True and d["ms_per_step"] > 0 and d["full_step_ms_extrapolated"] > 0


def test_config_is_identical_for_both_arms():
    import synth
    for name in ("tiny", "large"):
        w = synth.WORKLOADS[name]
        c = bench.workload_config(w, 1)
        assert c["n_active"] == bench.n_active_of(w)
    assert bench.workload_config(synth.WORKLOADS["large"], 1)["n_active"] == 18900


import pytest


@pytest.mark.gpu
def test_native_arm_prints_the_contract_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--steps", "3",
                        "--warmup", "3", "--no-cpu-baseline"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    from kv_cache_analyzer_b200.pipeline import KERNELS_PER_STEP
    # six of the library's kernels per step, one more when the attention's keys are split
    assert d["value"] > 0 and d["gpu_launches"] in (KERNELS_PER_STEP * 3, (KERNELS_PER_STEP + 1) * 3)
    assert d["config"] == bench.workload_config(synth.WORKLOADS["tiny"], 1)
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert r["traffic"] is None                  # the DRAM record belongs to the large workload
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
