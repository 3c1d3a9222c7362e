"""bench.py on a B200: the JSON line of each mode carries every field its readers need.

Small cases (a few million elements) so that each run takes seconds; the numbers themselves are
not checked here, only that they are present, finite and consistent.
"""
import json
import math
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.gpu
def test_default_line_fields():
    j = _run("--elements", "5120000", "--steps", "3", "--warmup", "3", "--e2e-steps", "1", "--cpu-seconds", "1")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in j, k
    assert j["n_gpus"] == 1 and j["steps"] == 3 and j["warmup"] == 3 and j["higher_is_better"] is True
    assert j["value"] > 0 and math.isfinite(j["value"]) and j["gpu_launches"] >= 3
    assert "workload" in j["config"] and "l2" in j["config"]
    r = j["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] < 2
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    c = j["cpu_baseline"]
    assert c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1 and c["sample"]
    e = j["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] == 8 * 4 * 5120000 and e["d2h_bytes_per_step"] == 4 * 5120000
    assert "sm_mhz" in j["clocks"] and "reasons" in j["clocks"]


@pytest.mark.gpu
def test_unfused_and_sweep_lines():
    u = _run("--unfused", "--elements", "5120000", "--steps", "2", "--warmup", "3")
    assert u["value"] > 0 and u["encode"]["frac"] > 0 and u["decode"]["frac"] > 0
    s = _run("--sweep", "--elements", "2097152", "--steps", "2", "--warmup", "3")
    rows = s["sweep"]
    assert {r["bucket"] for r in rows} == {128, 512, 2048, 8192, 32768}
    for r in rows:
        assert r["elem_per_s"] > 0 and 0 < r["normalised_variance"] < 10


@pytest.mark.gpu
def test_entropy_line():
    j = _run("--entropy", "--elements", "5120000", "--steps", "2", "--warmup", "3")
    assert j["value"] > 0 and j["pack"]["frac"] > 0 and j["unpack"]["frac"] > 0
    assert j["round_trip"] == "exact" and j["gpu_launches"] == 2 * 8 * 2
    c = j["compression"]
    # ORQ-5, d = 512: 38 words of codes per bucket against 48, plus the 5-float table
    assert abs(c["base_s_bits_per_elem"] - (38 * 32 + 5 * 32) / 512) < 1e-9
    assert abs(c["dense_bits_per_elem"] - (48 * 32 + 5 * 32) / 512) < 1e-9


@pytest.mark.gpu
def test_elias_line():
    j = _run("--elias", "--scheme", "qsgd_l2", "--levels", "3", "--elements", "5120000", "--steps", "2",
             "--warmup", "3")
    assert j["value"] > 0 and j["pack"]["frac"] > 0 and j["unpack"]["frac"] > 0
    assert j["round_trip"] == "exact" and j["gpu_launches"] == 6 * 8 * 2
    c = j["compression"]
    assert 1.0 <= c["stream_bits_per_elem"] < 1.3 and c["dense_bits_per_elem"] == (32 * 32 + 32) / 512


@pytest.mark.gpu
def test_exchange_line():
    """One rank: the all-gather is a copy on the GPU, no byte crosses a link."""
    j = _run("--exchange", "--elements", "5120000", "--steps", "2", "--warmup", "3")
    assert j["n_gpus"] == 1 and j["config"]["workers"] == 1 and j["value"] > 0
    assert j["encode"]["frac"] > 0 and j["decode"]["frac"] > 0
    assert j["allgather"]["bytes_received_per_rank"] == 0 and j["allgather"]["ms_per_call"] > 0
    assert j["gpu_launches"] == 2 * 2



@pytest.mark.gpu
def test_terngrad_layer_line():
    j = _run("--scheme", "terngrad_layer", "--workload", "resnet18", "--elements", "3000000", "--steps", "2",
             "--warmup", "3")
    assert j["value"] > 0 and j["config"]["tensors"] >= 2 and j["gpu_launches"] == 4
    r = j["roofline"]
    assert r["bound"] == "hbm" and 0 < r["frac"] < 2 and r["algorithmic_bytes_per_worker_elem"] > 20
