"""bench.py's output contract, checked without a GPU: the reference arm (the
fp64 oracle on the host) prints one JSON line with every required key, and
the host-side roofline arithmetic of the cross-attention field follows its
stated formulas."""

import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
         "--warmup", "1", "--workload", "tiny", "--cpu-rows", "64"],
        cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == "self-attn TFLOP/s" and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None
    assert d["data"] == "synthetic" and d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_cross_roofline_arithmetic():
    c = bench.cross_roofline(2, 1000, 4, 512, [100, 300], 2.0, 1000.0,
                             5000.0)
    flops = 4.0 * 1000 * 128 * 4 * (100 + 300)
    nbytes = 2.0 * 2 * 1000 * 4 * 256 + 2.0 * (100 + 300) * 4 * 256
    assert c["flops"] == flops and c["bytes"] == nbytes
    assert c["tflops"] == pytest.approx(flops / 2e-3 / 1e12)
    assert c["tflops_padded_lk"] == pytest.approx(
        4.0 * 2 * 1000 * 512 * 128 * 4 / 2e-3 / 1e12)
    assert c["gbs"] == pytest.approx(nbytes / 2e-3 / 1e9)
    assert c["frac_of_sustained_tensor_peak"] == pytest.approx(
        c["tflops"] / 1000.0)
    assert c["intensity_flop_per_byte"] == pytest.approx(flops / nbytes)
