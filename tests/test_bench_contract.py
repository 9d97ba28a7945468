"""bench.py's output contract: one JSON line with the keys the round driver
reads. The reference arm (the oracle, on the host) runs on CPU; our arm needs
a GPU."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=timeout, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--workload", "tiny_bf16", "--steps", "2", "--warmup", "1")
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_nvfp4_reference_arm_line():
    d = run_bench("--impl", "reference", "--workload", "nvfp4_t16384_k4096", "--steps", "1", "--warmup", "1")
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0


def test_smooth_reference_arm_line():
    d = run_bench("--impl", "reference", "--workload", "sage_k_smooth_s16384", "--steps", "1", "--warmup", "1")
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0


@pytest.mark.gpu
@pytest.mark.parametrize("workload", ["tiny_bf16", "decode_paged_s16384", "sage_k_smooth_s16384"])
def test_our_arm_line(workload):
    d = run_bench("--workload", workload, "--steps", "3", "--warmup", "3")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3 and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and 0 < r["frac"] < 1.5 and r["peak"] > 0
    assert d["config"]["workload"] and d["gpu_launches"] >= 3
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
