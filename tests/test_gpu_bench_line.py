"""The benchmark's JSON line on a B200: bench.py run as the driver runs it
(a child process), on the tiny workload and the activation-quantizer
configuration so that it takes seconds, and checked for every key and type
the line promises -- the metric and its unit, the timing fields, the
roofline, the CPU baseline, the end-to-end figure, the clock record and the
count of this library's kernel launches -- and for the reference arm's line."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-3000:]
    return json.loads(lines[0])


def _number(v):
    return isinstance(v, (int, float)) and not isinstance(v, bool)


def test_block_line_keys():
    d = _line("--workload", "tiny_w8a8_linear", "--steps", "10", "--warmup", "3", "--cpu-seconds", "0.5")
    for k in ("metric", "unit", "dtype", "data", "scaling"):
        assert isinstance(d[k], str) and d[k], k
    for k in ("value", "ms_per_step"):
        assert _number(d[k]) and d[k] > 0, k
    assert d["n_gpus"] == 1 and d["steps"] == 10 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == "tiny_w8a8_linear" and "not a benchmark" in d["config"]["l2"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and _number(r["achieved"]) and _number(r["peak"])
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3 and "traffic" in r
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and _number(c["value"]) and c["cores"] >= 1 and c["sample"]
    e = d["e2e"]
    assert _number(e["value"]) and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 64 * 256 * 2 and e["d2h_bytes_per_step"] == 64 * 128 * 2
    assert d["gpu_launches"] == 10 * 2  # one quantizer and one GEMM launch per step
    clk = d["clocks"]
    assert _number(clk["sm_mhz"]) and isinstance(clk["reasons"], list)


def test_quantizer_line_keys():
    d = _line("--workload", "activation_quantizer", "--steps", "5", "--warmup", "3", "--no-cpu-baseline")
    assert d["unit"] == "GB/s" and d["roofline"]["bound"] == "hbm" and _number(d["value"])
    assert d["gpu_launches"] == 5 * 2 and d["e2e"]["h2d_bytes_per_step"] == 8192 * 3072 * 2


def test_reference_arm_line():
    # one step of oracle work (about 15 s on the host cores) keeps the test short
    d = _line("--impl", "reference", "--workload", "tiny_w8a8_linear", "--steps", "1", "--warmup", "1")
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle" and _number(d["value"])
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
