"""The JSON line of bench.py: every key the benchmark contract asks for, with
values of the right kind, for the oracle arm (CPU) and the CUDA arm (GPU)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
             "scaling", "vs_baseline", "dtype", "data", "config"}


def _run(*args, timeout=600):
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.pop("RANK", None)
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout[-2000:]
    return json.loads(lines[0])


def _check_base(d, steps, warmup):
    assert BASE_KEYS <= set(d), BASE_KEYS - set(d)
    assert d["steps"] == steps and d["warmup"] == warmup and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["data"] == "synthetic" and d["vs_baseline"] is None
    assert "workload" in d["config"] and "flux_image" in d["config"]["workload"]


def test_reference_arm_line():
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "3")
    _check_base(d, 1, 3)
    assert d["impl"] == "reference" and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_own_arm_line():
    d = _run("--steps", "6", "--warmup", "3", "--warm-seconds", "0", "--no-secondary")
    _check_base(d, 6, 3)
    assert "impl" not in d and d["dtype"] == "bf16"
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
    assert r["traffic"] is None or r["traffic"] > 0
    c = d["clocks"]
    assert c["sm_mhz"] and c["sm_max_mhz"] and isinstance(c["reasons"], list)
    e = d["e2e"]
    assert e["unit"] == "TFLOP/s" and 0 < e["value"] <= d["value"]
    # Q, K, V in (bf16) and OUT, LSE out (fp32) of the flux_image step
    assert e["h2d_bytes_per_step"] == 3 * 24 * 4608 * 128 * 2
    assert e["d2h_bytes_per_step"] == 24 * 4608 * (128 + 1) * 4
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert d["gpu_launches"] == 6
