"""Host logic of bench.py on CPU: the clock record (NVML reason bits, the
summaries of NVML and nvidia-smi samples, a sampler run against a fake NVML
that offers only read calls), the traffic-record check and the step-floor
arithmetic of the path roofline."""
import sys
import time
import types

import pytest
import torch

import bench


def test_clock_reason_bits_match_nvml():
    pynvml = pytest.importorskip("pynvml")
    expect = {"sw_power_cap": "SwPowerCap", "hw_slowdown": "HwSlowdown",
              "sw_thermal_slowdown": "SwThermalSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
              "hw_power_brake_slowdown": "HwPowerBrakeSlowdown"}
    assert set(bench.CLOCK_REASON_BITS) == set(expect)
    for name, nv in expect.items():
        assert bench.CLOCK_REASON_BITS[name] == getattr(pynvml, "nvmlClocksThrottleReason" + nv)


def test_summarize_nvml_samples():
    samples = [(1200, 600.0, 0x4), (1300, 800.0, 0x4 | 0x1), (1250, 700.0, 0x0), (1260, 650.0, 0x10)]
    rec = bench.summarize_nvml_samples(samples, 1965.0, 1000.0)
    assert rec["sm_mhz"] == 1255 and rec["sm_max_mhz"] == 1965.0
    assert rec["power_w_max"] == 800.0 and rec["power_w_median"] == 675.0 and rec["power_limit_w"] == 1000.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] == 4   # idle (0x1), sync boost (0x10) unreported
    bad = bench.summarize_nvml_samples([(900, 500.0, 0x8 | 0x40), (950, 500.0, 0x20)], 1965.0, None)
    assert bad["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_nvml_samples([], 1965.0, 1000.0) is None
    # with the instantaneous board power (None where the field read failed)
    inst = bench.summarize_nvml_samples([(1200, 500.0, 0x4, 990.0), (1210, 520.0, 0x4, None),
                                         (1220, 540.0, 0x4, 1010.0), (1230, 560.0, 0x4, 1000.0)], 1965.0, 1000.0)
    assert inst["power_w_instant_median"] == 1000.0 and inst["power_w_instant_max"] == 1010.0
    assert inst["power_w_median"] == 530.0 and "power_note" in inst
    assert "power_w_instant_median" not in rec


def test_summarize_smi_lines():
    lines = ["0, 1245, 1965, 650.12, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
             "0, 1275, 1965, 700.50, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
             "0, [N/A], 1965, [N/A], 0x0, Not Active, Not Active, Not Active, Not Active\n",
             "truncated, line\n"]
    rec = bench.summarize_smi_lines(lines)
    assert rec["sm_mhz"] == 1260 and rec["sm_max_mhz"] == 1965.0 and rec["power_w_max"] == 700.5
    assert rec["samples"] == 3 and rec["reasons"] == ["sw_power_cap"]
    hot = bench.summarize_smi_lines(["0, 1000, 1965, 900, 0x48, Active, Active, Not Active, Not Active"])
    assert hot["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.summarize_smi_lines([]) is None


class _FakeNvml(types.ModuleType):
    """NVML with only the read calls the sampler may make; any other name
    (a setter, a reset) is missing, so using one fails the test."""
    NVML_CLOCK_SM = 1
    READS = {"nvmlInit", "nvmlDeviceGetHandleByPciBusId", "nvmlDeviceGetHandleByIndex", "nvmlDeviceGetClockInfo",
             "nvmlDeviceGetPowerUsage", "nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetMaxClockInfo",
             "nvmlDeviceGetEnforcedPowerLimit"}

    def __init__(self):
        super().__init__("pynvml")
        self.calls = []
        self.n = 0

    def _log(self, name):
        assert name in self.READS, name
        self.calls.append(name)

    def nvmlInit(self):
        self._log("nvmlInit")

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self._log("nvmlDeviceGetHandleByPciBusId")
        assert bus == "00000000:1b:00.0"
        return "handle"

    def nvmlDeviceGetHandleByIndex(self, i):
        self._log("nvmlDeviceGetHandleByIndex")
        return "handle"

    def nvmlDeviceGetClockInfo(self, h, kind):
        self._log("nvmlDeviceGetClockInfo")
        assert h == "handle" and kind == self.NVML_CLOCK_SM
        self.n += 1
        return 1200 + 100 * (self.n % 2)

    def nvmlDeviceGetPowerUsage(self, h):
        self._log("nvmlDeviceGetPowerUsage")
        return 650000  # milliwatts

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        self._log("nvmlDeviceGetCurrentClocksEventReasons")
        return 0x4

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        self._log("nvmlDeviceGetMaxClockInfo")
        return 1965

    def nvmlDeviceGetEnforcedPowerLimit(self, h):
        self._log("nvmlDeviceGetEnforcedPowerLimit")
        return 1000000


def test_sampler_reads_nvml_only(monkeypatch):
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1B, pci_device_id=0))
    s = bench.ClockSampler(0)
    assert s.nvml is not None
    s.start()
    deadline = time.time() + 10
    while len(s.samples) < 3 and time.time() < deadline:
        time.sleep(0.01)
    rec = s.stop()
    assert rec["source"] == "nvml, 10 ms" and rec["samples"] >= 3
    assert 1200 <= rec["sm_mhz"] <= 1300 and rec["sm_max_mhz"] == 1965.0
    assert rec["power_w_max"] == 650.0 and rec["power_limit_w"] == 1000.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert set(fake.calls) <= _FakeNvml.READS


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* header\n   comment */\nint f(int x) {\n\n  return x + 1;\n}\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b) != bench._code_only(c)


def test_recorded_traffic_only_while_sources_unchanged(monkeypatch, tmp_path):
    rec = tmp_path / "record.md"
    rec.write_text("text\n\n    workload = video_dit_block\n    dtype = fp8\n"
                   "    gemm.sources_sha256 = abc\n    gemm.traffic_bytes_per_launch = 1808000000\n")
    monkeypatch.setattr(bench, "traffic_record_path", lambda w, d: str(rec))
    monkeypatch.setattr(bench, "sources_sha256", lambda d, k: "abc")
    assert bench.recorded_traffic("gemm", "video_dit_block", "fp8") == 1808000000.0
    assert bench.recorded_traffic("quant", "video_dit_block", "fp8") is None      # no entry
    assert bench.recorded_traffic("gemm", "image_dit_block", "fp8") is None       # other workload
    monkeypatch.setattr(bench, "sources_sha256", lambda d, k: "def")
    assert bench.recorded_traffic("gemm", "video_dit_block", "fp8") is None       # kernel code changed


def test_hashed_sources_cover_every_included_header():
    """A traffic record's hash covers each kernel file and every header of the
    package it includes, directly or through another header."""
    import os
    import re
    csrc = os.path.join(bench.ROOT, bench._CSRC)
    for (dtype, kind), files in bench.KERNEL_SOURCES.items():
        todo, seen = list(files), set()
        while todo:
            f = todo.pop()
            if f in seen:
                continue
            seen.add(f)
            text = open(os.path.join(csrc, f), encoding="utf-8").read()
            todo += [h for h in re.findall(r'#include\s+"([^"]+)"', text) if os.path.exists(os.path.join(csrc, h))]
        assert seen == set(files), (dtype, kind, sorted(seen - set(files)))
        assert len(bench.sources_sha256(dtype, kind)) == 64


def test_path_roofline_floor():
    res = {"step_quant_bytes": [3e9, 1e9], "step_gemm_flops": [4e12, 1e12], "step_gemm_bytes": [2e9, 8e9],
           "ms_per_step": 5.0}
    peaks = {"hbm_gbs": 8000.0}
    out = bench.path_roofline(res, 1, peaks, 2000.0)
    # quantizers 4e9 B / 8e12 B/s = 0.5 ms; GEMM 1 compute bound 2.0 ms, GEMM 2 memory bound 1.0 ms
    assert out["floor_ms_measured_peaks"] == pytest.approx(3.5)
    assert out["frac_measured_peaks"] == pytest.approx(0.7)
    # at the 4.5 PFLOP/s spec GEMM 1 takes 4e12 / 4.5e15 s, still above its 0.25 ms of bytes
    assert out["floor_ms_spec"] == pytest.approx(0.5 + 1e3 * 4e12 / (bench.FP8_SPEC_TFLOPS * 1e12) + 1.0, rel=1e-4)


def test_profile_commands_still_run_with_this_bench(monkeypatch):
    """Every profile summary names the command that produced it: each
    `python bench.py ...` there parses with the bench's current options, and
    each ncu command leaves the GPU clocks alone (--clock-control none)."""
    import glob
    import os
    import shlex
    files = sorted(f for f in glob.glob(os.path.join(bench.ROOT, "profiles", "*.md"))
                   if os.path.basename(f) != "README.md")  # the index names no command
    assert files
    for f in files:
        text = open(f, encoding="utf-8").read().replace("\\\n", " ")
        cmds = [line.strip() for line in text.splitlines() if line.strip().startswith(("python bench.py", "ncu "))]
        assert any(c.startswith("ncu ") for c in cmds), f
        for c in cmds:
            if c.startswith("ncu ") and " -i " not in c:  # `ncu -i` reads a saved report: no GPU
                assert "--clock-control none" in c, (f, c)
            words = shlex.split(c)
            argv = words[words.index("bench.py"):] if "bench.py" in words else None
            if argv is not None:
                monkeypatch.setattr(sys, "argv", argv)
                bench.parse_args()  # exits (SystemExit) on an option the bench no longer has


def test_clock_normalised_fraction():
    """achieved / (SMs x 16384 FLOP/clk x sampled MHz); absent without a clock."""
    import bench
    r = bench.clock_normalised(2900.0, {"sm_mhz": 1230}, 148)
    peak = 148 * 16384 * 1230e6 / 1e12
    assert abs(r["peak_at_clock"] - round(peak, 1)) < 1e-9
    assert abs(r["frac"] - round(2900.0 / peak, 4)) < 1e-12
    assert bench.clock_normalised(2900.0, {}, 148) is None
    assert bench.clock_normalised(2900.0, {"sm_mhz": 1230}, None) is None


@pytest.mark.parametrize("M", [75600, 6889, 32760, 512, 129, 1])
def test_tile_sample_rows_hit_every_cta_share(M):
    """The full-size parity sample holds a row of every 128-row CTA share of
    M, the whole ragged last share, and the random rows."""
    import numpy as np
    from tests import _gpu
    rows = _gpu.tile_sample_rows(M, seed=3)
    assert rows.min() >= 0 and rows.max() < M and np.all(np.diff(rows) > 0)
    assert set(range(M - (M % 128 or min(M, 128)), M)) <= set(rows.tolist())
    assert len(rows) >= min(M, (M + 127) // 128 + 512) * 0.9
    with pytest.raises(AssertionError):
        _gpu.assert_covers_blocks(rows[rows >= 128], M) if M > 128 else _gpu.assert_covers_blocks(rows[:0], M)


def test_path_roofline_overlapped_floor():
    """A launch that quantizes inside its GEMM is floored at max(FLOPs / peak,
    (GEMM + quantizer bytes) / HBM); the serialized floor adds the quantizer's
    bytes / HBM to the GEMM's floor."""
    import bench
    hbm = 6543.1
    peaks = {"hbm_gbs": hbm}
    F, G, Q = 4e12, 1.2e9, 1.16e9
    res = {"ms_per_step": 2.0, "step_quant_bytes": [Q], "step_gemm_flops": [F, F], "step_gemm_bytes": [G, G],
           "step_ops": [("fused", F, G, Q), ("gemm", F, G, 0)]}
    out = bench.path_roofline(res, 1, peaks, 2800.0)
    t = lambda f, b: max(f / 2800e12, b / (hbm * 1e9))
    assert abs(out["floor_ms_measured_peaks"] - round(1e3 * (Q / (hbm * 1e9) + 2 * t(F, G)), 4)) < 1e-9
    assert abs(out["overlapped"]["floor_ms_measured_peaks"] - round(1e3 * (t(F, G + Q) + t(F, G)), 4)) < 1e-9
    res["step_ops"] = [("quant", 0, 0, Q), ("gemm", F, G, 0), ("gemm", F, G, 0)]
    assert "overlapped" not in bench.path_roofline(res, 1, peaks, 2800.0)


def test_clock_normalised_flags_short_regions():
    import bench
    r = bench.clock_normalised(2900.0, {"sm_mhz": 1965}, 148, region_ms=20.0)
    assert r["reliable"] is False and "too short" in r["note"]
    assert "reliable" not in bench.clock_normalised(2900.0, {"sm_mhz": 1230}, 148, region_ms=450.0)
