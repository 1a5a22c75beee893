"""The benchmark's JSON line: the keys and units the harness reads.

The reference arm (the oracle on the host cores) runs here on CPU on the
smallest workload; our arm needs a GPU and runs on a small workload too.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config", "e2e")


def _run(*args, timeout=900):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run("--impl", "reference", "--workload", "icl_n1k_m128_h4", "--steps", "2", "--warmup", "1",
             "--cpu-rows", "32")
    for key in BASE_KEYS + ("impl", "cpu_baseline"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "icl_n1k_m128_h4"


@pytest.mark.gpu
def test_our_arm_line():
    d = _run("--workload", "icl_n16k_m1k_h8", "--steps", "2", "--warmup", "3", "--cpu-rows", "32")
    for key in BASE_KEYS + ("roofline", "cpu_baseline", "clocks", "gpu_launches"):
        assert key in d, key
    assert d["unit"] == "TFLOP/s" and d["n_gpus"] == 1 and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0 and d["e2e"]["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["gpu_launches"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
    for name in ("icl_n1k_m128_h4", "icl_n16k_m1k_h8", "icl_n128k_m1k_h8_gated"):
        c = d["per_config"][name]
        assert 0 < c["attention_ms"]["min"] <= c["attention_ms"]["median"] <= c["attention_ms"]["p90"]
    assert d["parity_sample"]["within_gates"] and d["parity_sample"]["rows"] == 32
    assert 0 < d["parity_sample"]["vs_exact_rel_rms"] < 1
    assert d["cpu_baseline"]["one_thread"]["icl_n1k_m128_h4"]["tflops"] > 0
