#!/usr/bin/env python
"""Benchmark of the W8A8 scaled-FP8 Linear on B200.

A step is one pass of the whole hot path over one DiT block: for every
distinct activation of the block, per-token FP8 quantization (tfq kernel),
then every Linear reading it as a scaled FP8 GEMM with the fused
scale/bias/BF16 epilogue (tfq kernel; FP8 and INT8 run the Linears that
read one activation, Q, K and V, as one launch unless --separate).  Weights are quantized once per
channel before timing (the offline converter step).  The metric is the
block's GEMM FLOPs divided by the step time, which includes the activation
quantizers ("TFLOP/s incl. act quant").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle on a bounded sample

Prints ONE JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
each rank runs an independent replica of the workload (weak scaling, no
data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "scaled-FP8 Linear TFLOP/s incl. act quant, % of B200 FP8 dense peak"
FP8_SPEC_TFLOPS = 4500.0
FP8_OVER_BF16 = 2.0      # nominal dense ratio fp8 / bf16 (4.5 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


def metric_name(dtype: str) -> str:
    if dtype == "int8":
        return METRIC.replace("FP8", "INT8").replace("TFLOP/s", "TOPS")
    if dtype == "fp8_f16acc":
        return METRIC.replace("scaled-FP8 Linear", "scaled-FP8 Linear (FP16 accumulator)")
    if dtype == "mxfp8":
        return METRIC.replace("scaled-FP8 Linear", "MXFP8 Linear (E4M3, E8M0 scale per 32 values)")
    return METRIC


def unit_name(dtype: str) -> str:
    return "TOPS" if dtype == "int8" else "TFLOP/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="video_dit_block",
                    choices=["video_dit_block", "image_dit_block", "reduced_qmax_ffn_out", "tiny_w8a8_linear",
                             "activation_quantizer"],
                    help="activation_quantizer: X [8192, 3072] (1 %% outlier columns x50, 16 zero rows) quantized "
                         "per token to FP8 (448) and per row to INT8 (127); reports GB/s")
    ap.add_argument("--impl", default="tfq", choices=["tfq", "reference"])
    ap.add_argument("--dtype", default="fp8", choices=["fp8", "int8", "fp8_f16acc", "mxfp8"],
                    help="fp8: E4M3 W8A8 (the headline); int8: the INT8 W8A8 path; "
                         "fp8_f16acc: E4M3 with an FP16 accumulator; mxfp8: E4M3 with block-32 E8M0 scales")
    ap.add_argument("--fused", action="store_true",
                    help="fp8 only: the first Linear of each activation quantizes it inside its GEMM "
                         "(tfq_quant_scaled_fp8_linear: one kernel); the other Linears of that input take its codes")
    ap.add_argument("--separate", action="store_true",
                    help="FP8, INT8: one GEMM launch per Linear (by default the Linears that read one activation, "
                         "Q, K and V, run as one multi-Linear launch)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload's Linears over this many tokens instead of its M (for ncu captures on "
                         "a reduced case; never a benchmark figure)")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the e2e measurement (0: enough for about 0.5 s of copies)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-context", action="store_true", help="skip the torch._scaled_mm context line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


_CSRC = "int8_w8a8_quantized_b200/csrc/"
# Sources of the kernels a traffic record was captured on, per dtype and kind.
KERNEL_SOURCES = {
    ("fp8", "gemm"): ("tfq_gemm.cu", "tfq_gemm_common.cuh", "tfq_ptx.cuh", "tfq_internal.h", "tfq_quant_row.cuh",
                      "tfq_quant_common.cuh"),
    ("fp8", "quant"): ("tfq_quant.cu", "tfq_quant_common.cuh", "tfq_quant_row.cuh", "tfq_ptx.cuh", "tfq_internal.h"),
    ("int8", "gemm"): ("tfq_gemm.cu", "tfq_gemm_common.cuh", "tfq_ptx.cuh", "tfq_internal.h", "tfq_quant_row.cuh",
                       "tfq_quant_common.cuh"),
    ("int8", "quant"): ("tfq_quant.cu", "tfq_quant_common.cuh", "tfq_quant_row.cuh", "tfq_ptx.cuh", "tfq_internal.h"),
    ("fp8_f16acc", "gemm"): ("tfq_gemm.cu", "tfq_gemm_common.cuh", "tfq_ptx.cuh", "tfq_internal.h",
                             "tfq_quant_row.cuh", "tfq_quant_common.cuh"),
    ("fp8_f16acc", "quant"): ("tfq_quant.cu", "tfq_quant_common.cuh", "tfq_quant_row.cuh", "tfq_ptx.cuh",
                              "tfq_internal.h"),
    ("mxfp8", "gemm"): ("tfq_gemm_mx.cu", "tfq_gemm_common.cuh", "tfq_ptx.cuh", "tfq_internal.h"),
    ("mxfp8", "quant"): ("tfq_quant_mx.cu", "tfq_quant_common.cuh", "tfq_ptx.cuh", "tfq_internal.h"),
}


def traffic_record_path(workload: str, dtype: str) -> str:
    suffix = "" if dtype == "fp8" else f"_{dtype}"
    return os.path.join(ROOT, "profiles", f"roofline_traffic_{workload}{suffix}.md")


TRAFFIC_RECORD = traffic_record_path("video_dit_block", "fp8")


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and blank lines (the kernels'
    sources hold no '//' or '/*' inside string literals)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def sources_sha256(dtype: str, kind: str) -> str:
    """SHA-256 of the code (comments stripped) of the sources of a dtype's
    kernels: a traffic record stays valid while that code is unchanged."""
    import hashlib
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[(dtype, kind)]:
        with open(os.path.join(ROOT, _CSRC + f), encoding="utf-8") as fh:
            m.update(_code_only(fh.read()).encode())
    return m.hexdigest()


def recorded_traffic(kind: str, workload: str, dtype: str):
    """DRAM bytes per launch from the committed ncu capture of this workload and
    dtype (profiles/roofline_traffic_<workload>[_<dtype>].md), or None when there
    is none or the kernel sources changed since it was taken."""
    try:
        kv = {}
        for line in open(traffic_record_path(workload, dtype), encoding="utf-8"):
            if " = " in line:
                k, v = line.strip().split(" = ", 1)
                kv[k] = v
        if kv.get("workload") != workload or kv.get("dtype") != dtype:
            return None
        if sources_sha256(dtype, kind) != kv.get(f"{kind}.sources_sha256"):
            return None
        return float(kv[f"{kind}.traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed region:
    through NVML every 10 ms from a background thread (so that even a timed
    region of a few milliseconds has samples), else nvidia-smi every 200 ms."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.nvml = None
        self.thread = None
        self.samples = []
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            handle = None
            props = torch.cuda.get_device_properties(gpu_index)
            try:  # the NVML device with this CUDA device's PCI address
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.nvml = (pynvml, handle)
        except Exception:
            self.nvml = None

    def _poll(self):
        import time as _t
        pynvml, h = self.nvml
        reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        fid = getattr(pynvml, "NVML_FI_DEV_POWER_INSTANT", None)
        while not self.stop_flag:
            try:
                inst = None
                if fid is not None:  # the board's instantaneous power (read only)
                    try:
                        fv = pynvml.nvmlDeviceGetFieldValues(h, [fid])[0]
                        if fv.nvmlReturn == 0:
                            inst = float(fv.value.uiVal) / 1000.0
                    except Exception:
                        fid = None
                self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons_fn(h)), inst))
            except Exception:
                pass
            _t.sleep(0.01)

    def start(self):
        if self.nvml is not None:
            import threading
            self.stop_flag = False
            self.samples = []
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            self.thread = None
            pynvml, h = self.nvml
            try:
                sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            except Exception:
                sm_max = None
            try:  # read only: the enforced board power limit sets the clock a power-bound kernel gets
                limit_w = pynvml.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
            except Exception:
                limit_w = None
            return summarize_nvml_samples(self.samples, sm_max, limit_w)
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as fh:
            lines = fh.readlines()
        os.unlink(self.path)
        return summarize_smi_lines(lines)


# NVML clock-event reason bits (nvmlClocksEventReason*) reported by name.
CLOCK_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                     "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


def summarize_nvml_samples(samples, sm_max, limit_w):
    """Clock record from NVML samples (SM MHz, board watts as NVML's power
    usage, reason bit mask[, instantaneous board watts or None]): median SM
    clock and power, the peak power, and every reason that was active in any
    sample.  None without samples."""
    if not samples:
        return None
    reasons = sorted(n for n, bit in CLOCK_REASON_BITS.items() if any(smp[2] & bit for smp in samples))
    rec = {"sm_mhz": statistics.median(smp[0] for smp in samples), "sm_max_mhz": sm_max,
           "power_w_max": max(smp[1] for smp in samples),
           "power_w_median": statistics.median(smp[1] for smp in samples),
           "power_limit_w": limit_w, "samples": len(samples),
           "source": "nvml, 10 ms", "reasons": reasons}
    inst = [smp[3] for smp in samples if len(smp) > 3 and smp[3] is not None]
    if inst:
        rec["power_w_instant_median"] = statistics.median(inst)
        rec["power_w_instant_max"] = max(inst)
        rec["power_note"] = ("power_w_median/max: NVML power usage, averaged by the driver over a window that "
                             "lags a short timed region; power_w_instant_*: the instantaneous board power")
    return rec


def summarize_smi_lines(lines):
    """Clock record from `nvidia-smi --query-gpu=ClockSampler.QUERY
    --format=csv,noheader,nounits` lines; a reason counts when any sample
    shows it "Active".  None without a complete line."""
    rows = [parts for parts in ([p.strip() for p in line.split(",")] for line in lines) if len(parts) >= 9]
    if not rows:
        return None

    def num(v):
        try:
            return float(v)
        except ValueError:
            return None
    sm = [num(r[1]) for r in rows if num(r[1]) is not None]
    pw = [num(r[3]) for r in rows if num(r[3]) is not None]
    reasons = set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        for name, v in zip(names, r[5:9]):
            if v.strip().lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": num(rows[0][2]),
            "power_w_max": max(pw) if pw else None,
            "samples": len(rows),
            "source": "nvidia-smi, 200 ms",
            "reasons": sorted(reasons)}


# --------------------------------------------------------- multi-rank
def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank timing over all ranks (the only collective: plumbing,
    not data path).  `device` is where the backend wants the tensor."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(world: int, flops_per_step: int, ms_per_step_max: float) -> float:
    """Whole-job TFLOP/s: every rank runs one replica of the workload per
    step (weak scaling), timed by the slowest rank."""
    return world * flops_per_step / (ms_per_step_max * 1e-3) / 1e12


# ------------------------------------------------------------ GPU arm
def step_working_set_bytes(wl) -> int:
    """Bytes one step touches: the bf16 activations, the 8-bit weights and the
    bf16 outputs of every Linear (codes and scales of the activations aside)."""
    xs = sum(wl.M * k * 2 for k in wl.x_shapes().values())
    return xs + sum(lin.N * lin.K + 2 * wl.M * lin.N for lin in wl.linears) * len(wl.act_qmax)


def l2_note(wl) -> str:
    """How the timing treats L2 (126 MB): no flush where every activation is
    larger than L2 or where one step's working set is; otherwise say that the
    workload fits (a parity-size case, not a benchmark figure)."""
    if wl.M * min(l.K for l in wl.linears) * 2 > L2_BYTES:
        return "inputs larger than L2 (126 MB)"
    ws = step_working_set_bytes(wl)
    if ws > L2_BYTES:
        return f"working set of one step ({ws / 1e6:.0f} MB) larger than L2; no flush"
    return f"working set of one step ({ws / 1e6:.1f} MB) fits in L2, not flushed: a parity-size case, not a benchmark"


def act_qmaxes(wl, dtype):
    """Activation quantization passes per step: one per qmax; INT8 uses 127,
    MXFP8 has no qmax (its scale comes from each block's exponent), and the
    FP16-accumulator GEMM takes activations quantized with qmax 7 -- the DiT
    setting the LightX2V page pairs with FP16 accumulation; at 448 (and at 14
    on the FFN-out shape) its partial sums overflow FP16."""
    if dtype == "int8":
        return (127.0,)
    if dtype == "mxfp8":
        return (0.0,)
    if dtype == "fp8_f16acc":
        return (7.0,)
    return wl.act_qmax


def build_block(wl, dev, dtype="fp8"):
    """Device-resident inputs, quantized weights and outputs of one block."""
    import torch
    from int8_w8a8_quantized_b200 import tfq_quant_weight_per_channel

    from int8_w8a8_quantized_b200 import tfq_mxfp8_scale_bytes, tfq_quant_mxfp8
    xs = {name: wl.make_x(name, device=dev) for name in sorted(wl.x_shapes())}
    lins = []
    for lin in wl.linears:
        w = wl.make_w(lin, device=dev)
        if dtype == "mxfp8":
            Wq, sw = tfq_quant_mxfp8(w)
        else:
            wdt = "int8" if dtype == "int8" else "fp8"
            Wq, sw = tfq_quant_weight_per_channel(w, wdt, 127.0 if dtype == "int8" else 448.0)
        del w
        b = wl.make_bias(lin, device=dev)
        lins.append((lin, Wq, sw, b))

    def act_scales(x):
        if dtype == "mxfp8":  # E8M0 codes in the tensor-core scale layout
            return torch.empty(tfq_mxfp8_scale_bytes(x.shape[0], x.shape[1]), dtype=torch.uint8, device=dev)
        return torch.empty(x.shape[0], device=dev)
    aq = {(name, q): (torch.empty_like(x, dtype=torch.uint8), act_scales(x))
          for name, x in xs.items() for q in act_qmaxes(wl, dtype)}
    ys = {(lin.name, q): torch.empty((wl.M, lin.N), dtype=torch.bfloat16, device=dev)
          for lin in wl.linears for q in act_qmaxes(wl, dtype)}
    torch.cuda.synchronize()
    return xs, lins, aq, ys


def gpu_arm(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from int8_w8a8_quantized_b200 import _capi

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = _capi.load_library()
    stream = torch.cuda.current_stream()
    sh = int(stream.cuda_stream)
    xs, lins, aq, ys = build_block(wl, dev, args.dtype)
    qmaxes = act_qmaxes(wl, args.dtype)
    if args.dtype == "mxfp8":
        def quant_fn(x, M, K, q, A, sf, s):
            return lib.tfq_quant_mxfp8(x, M, K, A, sf, s)
    else:
        quant_fn = lib.tfq_quant_act_int8_per_token if args.dtype == "int8" else lib.tfq_quant_act_fp8_per_token
    gemm_fn = {"fp8": lib.tfq_scaled_fp8_linear, "int8": lib.tfq_scaled_int8_linear,
               "fp8_f16acc": lib.tfq_scaled_fp8_linear_f16acc, "mxfp8": lib.tfq_mxfp8_linear}[args.dtype]
    mx = args.dtype == "mxfp8"

    # per-kernel events, recorded on the launching stream
    ev = {"quant": [], "gemm": [], "fused": []}
    launches = [0]

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {_capi.status_string(st)}: {_capi.last_error_message()}")

    # One step's launches in order: (kind, launch, metadata).  Kinds: "quant"
    # (a row quantizer; metadata = algorithmic bytes: read bf16, write 8-bit
    # codes, 4 B of scale per row or, MXFP8, 1 B per 32 values), "gemm" (a
    # GEMM on quantized operands; metadata = (M, N, K)) and, with --fused,
    # "fused" (the first Linear of each activation quantizes it inside its
    # GEMM; metadata = (M, N, K, quantizer bytes)).
    fused = getattr(args, "fused", False)
    multi = getattr(args, "multi", False)
    multi_fn = lib.tfq_scaled_int8_linear_multi if args.dtype == "int8" else lib.tfq_scaled_fp8_linear_multi

    def multi_arrays(group, q, outs=None):
        """The array arguments of the multi-Linear GEMM for the Linears of
        `group` (weights, scales, biases, N, outputs from `outs`, default the
        block's outputs) and the stream."""
        outs = ys if outs is None else outs
        return (_capi.pointer_array([W.data_ptr() for _, W, _, _ in group]),
                _capi.pointer_array([s.data_ptr() for _, _, s, _ in group]),
                _capi.pointer_array([None if bb is None else bb.data_ptr() for _, _, _, bb in group]),
                (ctypes.c_int64 * len(group))(*[l.N for l, _, _, _ in group]),
                _capi.pointer_array([outs[(l.name, q)].data_ptr() for l, _, _, _ in group]), sh)
    wss = {name: torch.empty(lib.tfq_quant_scaled_fp8_linear_workspace_bytes(x.shape[0]), dtype=torch.uint8,
                             device=dev) for name, x in xs.items()} if fused else {}
    ops = []
    quant_inputs = {}  # op index -> the activation a quantizer launch reads
    # Block order, as a LinearFP8 forward runs: each activation is quantized
    # directly before the first Linear that reads it (Q, K and V share theirs).
    for q in qmaxes:
        seen = set()
        for lin, Wq, sw, b in lins:
            A, sa = aq[(lin.x, q)]
            y = ys[(lin.name, q)]
            bp = None if b is None else b.data_ptr()
            if not fused and lin.x not in seen:
                x = xs[lin.x]
                quant_inputs[len(ops)] = x
                ops.append(("quant",
                            lambda x=x, q=q, A=A, sa=sa: quant_fn(x.data_ptr(), x.shape[0], x.shape[1], float(q),
                                                                  A.data_ptr(), sa.data_ptr(), sh),
                            3 * x.numel() + (x.numel() // 32 if mx else 4 * x.shape[0])))
            if fused and lin.x not in seen:
                x = xs[lin.x]
                ops.append(("fused",
                            lambda x=x, q=q, Wq=Wq, sw=sw, bp=bp, lin=lin, A=A, sa=sa, y=y, ws=wss[lin.x]:
                            lib.tfq_quant_scaled_fp8_linear(x.data_ptr(), wl.M, lin.K, float(q), Wq.data_ptr(),
                                                            sw.data_ptr(), bp, lin.N, A.data_ptr(), sa.data_ptr(),
                                                            y.data_ptr(), ws.data_ptr(), sh),
                            (wl.M, lin.N, lin.K, 3 * x.numel() + 4 * x.shape[0])))
            elif multi and lin.x in seen:
                pass  # launched with the first Linear that reads lin.x
            elif multi:
                group = [(l, W, s, bb) for l, W, s, bb in lins if l.x == lin.x]
                arrs = multi_arrays(group, q)
                ops.append(("gemm",
                            lambda A=A, sa=sa, lin=lin, n=len(group), arrs=arrs:
                            multi_fn(A.data_ptr(), sa.data_ptr(), wl.M, lin.K, n, *arrs),
                            (wl.M, sum(l.N for l, _, _, _ in group), lin.K)))
            else:
                ops.append(("gemm",
                            lambda A=A, sa=sa, Wq=Wq, sw=sw, bp=bp, lin=lin, y=y:
                            gemm_fn(A.data_ptr(), sa.data_ptr(), Wq.data_ptr(), sw.data_ptr(), bp, wl.M, lin.N,
                                    lin.K, y.data_ptr(), sh),
                            (wl.M, lin.N, lin.K)))
            seen.add(lin.x)
    n_kernels = len(ops)

    def step(record, which=None):
        """One block step; with `record`, CUDA events bracket kernel `which` of
        the step (every kernel when which is None)."""
        for k, (kind, launch, meta) in enumerate(ops):
            rec = record and (which is None or k == which)
            if rec:
                e0 = torch.cuda.Event(enable_timing=True); e0.record(stream)
            check(launch(), kind)
            launches[0] += 1
            if rec:
                e1 = torch.cuda.Event(enable_timing=True); e1.record(stream)
                ev[kind].append((e0, e1, meta))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    check(lib.tfq_device_error(sh), "device error after warm-up")

    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches[0] = 0
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    # Per-kernel events: step i brackets kernel i mod n_kernels only, so that every kernel is timed
    # in steps / n_kernels of the steps and the other kernel boundaries run as they would without a
    # profiler (an event between two kernels serialises their launches).  Fewer steps than kernels:
    # events around every kernel of every step.
    sample_one = args.steps >= n_kernels
    for i in range(args.steps):
        step(True, (i % n_kernels) if sample_one else None)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    check(lib.tfq_device_error(sh), "device error in the timed region")
    ms = max_over_ranks(t0.elapsed_time(t1), dev) if world > 1 else t0.elapsed_time(t1)
    ms_per_step = ms / args.steps

    # What the step allows a stream of the quantizers' bytes: the same step with
    # every quantizer launch replaced by a device copy of the same traffic (it
    # reads and writes half of the launch's algorithmic bytes each), in its
    # place between the GEMMs, timed the same way.  Context for quantizer.frac
    # (the achievable bandwidth at the clock the GEMMs leave), not part of the metric.
    copy_ref = None
    if quant_inputs:
        nbs = {k: ops[k][2] // 2 for k in quant_inputs}
        dst = torch.empty(max(nbs.values()), dtype=torch.uint8, device=dev)
        copy_ops = []
        for k, (kind, launch, meta) in enumerate(ops):
            if k in quant_inputs:
                src = quant_inputs[k].view(-1).view(torch.uint8)[:nbs[k]]
                copy_ops.append(("copy", lambda s=src, d=dst[:nbs[k]]: d.copy_(s), 2 * nbs[k]))
            else:
                copy_ops.append((kind, launch, meta))
        cev = []
        for i in range(2 + args.steps):
            for k, (kind, launch, meta) in enumerate(copy_ops):
                rec = i >= 2 and kind == "copy" and (k == i % len(copy_ops) or not sample_one)
                if rec:
                    e0 = torch.cuda.Event(enable_timing=True); e0.record(stream)
                if kind == "copy":
                    launch()
                else:
                    check(launch(), kind)
                if rec:
                    e1 = torch.cuda.Event(enable_timing=True); e1.record(stream)
                    cev.append((e0, e1, meta))
        torch.cuda.synchronize()
        if cev:
            cms = sum(a.elapsed_time(b) for a, b, _ in cev)
            copy_ref = {"gbs": sum(m for _, _, m in cev) / (cms * 1e-3) / 1e9, "launches_timed": len(cev),
                        "what": "the step with each quantizer launch replaced by a device copy of the same "
                                "traffic (half read, half written), events as for the quantizers"}
        del dst

    # one step's kernels (for the path floor), independent of which launches had events
    step_shapes = [meta[:3] for kind, _, meta in ops if kind != "quant"]
    step_quant_bytes = [3 * x.numel() + (x.numel() // 32 if mx else 4 * x.shape[0]) for q in qmaxes for x in xs.values()]

    def gemm_step_bytes(m, n, k):
        # codes, scales (MXFP8: 1 B per 32 values of each operand), bf16 output, bias
        return m * k + n * k + ((m + n) * k // 32 + 2 * m * n + 2 * n if mx else 2 * m * n + 4 * m + 6 * n)
    gemm_ms = [a.elapsed_time(b) for a, b, _ in ev["gemm"]]
    quant_ms = [a.elapsed_time(b) for a, b, _ in ev["quant"]]
    fused_ms = [a.elapsed_time(b) for a, b, _ in ev["fused"]]
    gemm_flops = [2 * m * n * k for _, _, (m, n, k) in ev["gemm"]]
    gemm_bytes = [gemm_step_bytes(m, n, k) for _, _, (m, n, k) in ev["gemm"]]
    quant_bytes = [nbytes for _, _, nbytes in ev["quant"]]
    out = {
        "ms_per_step": ms_per_step,
        "step_gemm_flops": [2 * m * n * k for m, n, k in step_shapes],
        "step_gemm_bytes": [gemm_step_bytes(m, n, k) for m, n, k in step_shapes],
        "step_quant_bytes": step_quant_bytes,
        # every launch of a step: (kind, FLOPs, GEMM bytes, quantizer bytes)
        "step_ops": [(kind, 0, 0, meta) if kind == "quant" else
                     (kind, 2 * meta[0] * meta[1] * meta[2], gemm_step_bytes(*meta[:3]),
                      meta[3] if kind == "fused" else 0) for kind, _, meta in ops],
        "gemm_ms_total": sum(gemm_ms), "gemm_flops_total": sum(gemm_flops), "gemm_bytes_total": sum(gemm_bytes),
        "quant_ms_total": sum(quant_ms), "quant_bytes_total": sum(quant_bytes),
        "fused_ms_total": sum(fused_ms),
        "fused_flops_total": sum(2 * m * n * k for _, _, (m, n, k, _) in ev["fused"]),
        "fused_bytes_total": sum(gemm_step_bytes(m, n, k) + qb for _, _, (m, n, k, qb) in ev["fused"]),
        "fused_launches": len(fused_ms),
        "gemm_launches": len(gemm_ms), "quant_launches": len(quant_ms),
        "quant_launches_per_step": sum(1 for kind, _, _ in ops if kind == "quant"),
        "kernel_events": (f"each kernel bracketed in {args.steps // n_kernels}-{-(-args.steps // n_kernels)} of "
                          f"the {args.steps} timed steps (one kernel per step)") if sample_one
        else "every kernel of every timed step",
        "gpu_launches": launches[0], "clocks": clk, "quant_copy_reference": copy_ref,
        "sm_count": torch.cuda.get_device_properties(dev).multi_processor_count,
        "per_linear": {},
    }
    for (a, b, meta) in ev["gemm"] + ev["fused"]:
        key = "x".join(str(v) for v in meta[:3]) + (" (quantizing)" if len(meta) == 4 else "")
        out["per_linear"].setdefault(key, []).append(a.elapsed_time(b))

    # outputs of the last timed step that are not finite (an FP16 accumulator can overflow); outside the timing
    out["nonfinite_outputs"] = int(sum(int((~torch.isfinite(y)).sum()) for y in ys.values()))
    out["context"] = torch_scaled_mm_context(args, wl, lins, aq, ys, qmaxes, stream) if not args.no_context else None

    # -------- end-to-end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = e2e_arm(args, wl, qmaxes, quant_fn, gemm_fn, xs, lins, aq, ys, stream, sh, check, lib=lib,
                      wss=wss if fused else None, multi=(multi_fn, multi_arrays) if multi else None)
    return out, e2e


def torch_scaled_mm_context(args, wl, lins, aq, ys, qmaxes, stream):
    """Context line, outside the timed region: the block's GEMMs through
    torch._scaled_mm (cuBLASLt; row-wise fp32 scales, bias, bf16 out) on the same
    quantized operands, CUDA events per call after two warm-up calls.  FP8 only."""
    import torch
    if args.dtype not in ("fp8", "fp8_f16acc"):
        return None
    try:
        flops = 0
        ms = 0.0
        per = {}
        for q in qmaxes:
            for lin, Wq, sw, b in lins:
                A, sa = aq[(lin.x, q)]
                a8, w8 = A.view(torch.float8_e4m3fn), Wq.view(torch.float8_e4m3fn)

                def call():
                    return torch._scaled_mm(a8, w8.t(), scale_a=sa.view(-1, 1), scale_b=sw.view(1, -1), bias=b,
                                            out_dtype=torch.bfloat16)
                for _ in range(2):
                    call()
                times = []
                for _ in range(3):
                    e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream); r = call(); e1.record(stream)
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1))
                    del r
                t = statistics.median(times)
                ms += t
                flops += 2 * wl.M * lin.N * lin.K
                per[f"{wl.M}x{lin.N}x{lin.K}"] = round(t, 4)
        return {"torch_scaled_mm_tflops": round(flops / (ms * 1e-3) / 1e12, 1), "per_linear_ms": per,
                "what": "the block's GEMMs through torch._scaled_mm (cuBLASLt, row-wise fp32 scales, bias, bf16 "
                        "out) on the same quantized operands; median of 3 calls each, outside the timed region"}
    except Exception as e:  # a torch build without FP8 scaled_mm on this device
        return {"error": f"{type(e).__name__}: {str(e)[:200]}"}


def e2e_arm(args, wl, qmaxes, quant_fn, gemm_fn, xs, lins, aq, ys, stream, sh, check, lib=None, wss=None,
            multi=None):
    """Every step: H2D copy of each activation of the block from pinned host
    memory, the quantizers and GEMMs, D2H copy of every output into pinned
    host memory.  The copies run on two copy streams and overlap the
    compute stream; the device buffers (activations, codes, outputs) are
    double-buffered, steps alternating between the two sets, so that a
    step's H2D copies overlap the previous step's kernels and D2H copies.
    Events order each copy with the kernels that produce or consume its
    buffer, also across steps; the timed region ends when the last D2H copy
    has landed."""
    import torch
    hx = {n: torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for n, x in xs.items()}
    for n, x in xs.items():
        hx[n].copy_(x)
    hy = {k: torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for k, y in ys.items()}
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in hy.values())
    # the second device set
    sets = [(xs, aq, ys),
            ({n: torch.empty_like(x) for n, x in xs.items()},
             {k: tuple(torch.empty_like(t) for t in v) for k, v in aq.items()},
             {k: torch.empty_like(y) for k, y in ys.items()})]
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    order = []  # activations in the order the block uses them
    for lin in lins:
        if lin[0].x not in order:
            order.append(lin[0].x)
    multi_fn, multi_arrays = multi if multi is not None else (None, None)
    x_read = {}   # (set, x): event, the quantizers of the set's previous step finished reading x
    y_read = {}   # (set, y): event, the D2H copy of the set's previous step finished reading y
    counter = [0]

    def step():
        k = counter[0] % 2
        counter[0] += 1
        xk, aqk, ysk = sets[k]
        landed = {}
        for n in order:
            if (k, n) in x_read:
                copy_in.wait_event(x_read[(k, n)])
            with torch.cuda.stream(copy_in):
                xk[n].copy_(hx[n], non_blocking=True)
            landed[n] = torch.cuda.Event()
            landed[n].record(copy_in)

        def to_host(key):
            with torch.cuda.stream(copy_out):
                hy[key].copy_(ysk[key], non_blocking=True)
            y_read[(k, key)] = torch.cuda.Event()
            y_read[(k, key)].record(copy_out)

        for n in order:
            stream.wait_event(landed[n])
            x = xk[n]
            if wss is None:
                for q in qmaxes:
                    A, sa = aqk[(n, q)]
                    check(quant_fn(x.data_ptr(), x.shape[0], x.shape[1], float(q), A.data_ptr(), sa.data_ptr(),
                                   sh), "quant")
                x_read[(k, n)] = torch.cuda.Event()
                x_read[(k, n)].record(stream)
            for q in qmaxes:
                A, sa = aqk[(n, q)]
                first = True
                if multi_fn is not None:  # the Linears that read x as one launch
                    group = [(lin, Wq, sw, b) for lin, Wq, sw, b in lins if lin.x == n]
                    for lin, _, _, _ in group:
                        if (k, (lin.name, q)) in y_read:
                            stream.wait_event(y_read[(k, (lin.name, q))])
                    check(multi_fn(A.data_ptr(), sa.data_ptr(), wl.M, group[0][0].K, len(group),
                                   *multi_arrays(group, q, ysk)), "gemm")
                    done = torch.cuda.Event()
                    done.record(stream)
                    copy_out.wait_event(done)
                    for lin, _, _, _ in group:
                        to_host((lin.name, q))
                    continue
                for lin, Wq, sw, b in lins:
                    if lin.x != n:
                        continue
                    key = (lin.name, q)
                    y = ysk[key]
                    if (k, key) in y_read:
                        stream.wait_event(y_read[(k, key)])
                    bp = None if b is None else b.data_ptr()
                    if wss is not None and first:  # quantizes x inside its GEMM
                        check(lib.tfq_quant_scaled_fp8_linear(x.data_ptr(), wl.M, lin.K, float(q), Wq.data_ptr(),
                                                              sw.data_ptr(), bp, lin.N, A.data_ptr(), sa.data_ptr(),
                                                              y.data_ptr(), wss[n].data_ptr(), sh), "fused")
                        if q == qmaxes[-1]:
                            x_read[(k, n)] = torch.cuda.Event()
                            x_read[(k, n)].record(stream)
                    else:
                        check(gemm_fn(A.data_ptr(), sa.data_ptr(), Wq.data_ptr(), sw.data_ptr(), bp, wl.M, lin.N,
                                      lin.K, y.data_ptr(), sh), "gemm")
                    first = False
                    done = torch.cuda.Event()
                    done.record(stream)
                    copy_out.wait_event(done)
                    to_host(key)

    # Floor of the step over PCIe: the same copies with no kernels, both
    # directions at once on the same two copy streams (same buffers, same
    # bytes; the contents written are the ones already there).
    def copies_only():
        copy_in.wait_stream(stream)
        copy_out.wait_stream(stream)
        with torch.cuda.stream(copy_in):
            for n in order:
                xs[n].copy_(hx[n], non_blocking=True)
        with torch.cuda.stream(copy_out):
            for key, y in ys.items():
                hy[key].copy_(y, non_blocking=True)
        stream.wait_stream(copy_in)
        stream.wait_stream(copy_out)

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)

    def timed(fn, n):
        torch.cuda.synchronize()
        t0.record(stream)
        copy_in.wait_stream(stream)  # no copy of the timed steps starts before t0
        copy_out.wait_stream(stream)
        for _ in range(n):
            fn()
        stream.wait_stream(copy_out)
        stream.wait_stream(copy_in)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n

    copies_only()
    # Steps timed: --e2e-steps, or (0, the default) enough for about 0.5 s of
    # copies, so that filling and draining the copy pipeline (the first H2D
    # before any kernel, the last D2H after them) is a small part of the region.
    n_steps = args.e2e_steps or max(3, min(200, math.ceil(500.0 / max(timed(copies_only, 2), 1e-3))))
    copy_ms = timed(copies_only, n_steps)
    step()
    step()  # both device sets once before timing
    ms = timed(step, n_steps)
    flops = wl.flops() // len(wl.act_qmax) * len(qmaxes)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": unit_name(args.dtype), "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_steps,
            "host_buffers": "pinned",
            "overlap": "H2D and D2H on two copy streams, overlapping compute; device buffers double-buffered",
            "copies_alone_ms": round(copy_ms, 3), "frac_of_copy_floor": round(copy_ms / ms, 4),
            "floor": "the step's H2D and D2H copies alone, both directions at once, no kernels"}


# ------------------------------------------------------------ CPU oracle
def oracle_sample(wl, seconds: float, seed: int = 0, dtype: str = "fp8"):
    """Runs the oracle (quantizer + double GEMM) on a bounded sample of the
    workload's rows; returns (flops_done, seconds_taken, description)."""
    import numpy as np
    import torch
    import oracle

    rng = np.random.default_rng(seed)
    # Rows are independent, so a sample of rows is a sample of the job: each
    # pass quantizes `threads` fresh rows per Linear (drawn with the same
    # recipe) and multiplies them by the full per-channel FP8 weight, which
    # keeps every OpenMP thread of the oracle busy.
    rows_per_linear = oracle.num_threads()
    total_flops = 0
    t_total = 0.0
    done = []
    cache = {}
    while t_total < seconds:
        for lin in wl.linears:
            key = lin.name
            if key not in cache:
                w = wl.make_w(lin)
                wbits = w.contiguous().view(torch.int16).numpy().view(np.uint16)
                if dtype == "mxfp8":
                    Wq, sw = oracle.quant_mxfp8(wbits)
                else:
                    Wq, sw = oracle.quant_rows_int8(wbits) if dtype == "int8" else oracle.quant_rows_fp8(wbits, 448.0)
                b = wl.make_bias(lin)
                bbits = None if b is None else b.contiguous().view(torch.int16).numpy().view(np.uint16)
                cache[key] = (Wq, sw, bbits)
            Wq, sw, bbits = cache[key]
            x = _x_rows(wl, lin, rows_per_linear, int(rng.integers(1 << 30)))
            for q in act_qmaxes(wl, dtype):
                t0 = time.perf_counter()
                if dtype == "mxfp8":
                    A, sa = oracle.quant_mxfp8(x)
                    oracle.mxfp8_linear(A, sa, Wq, sw, bbits)
                elif dtype != "int8":  # the oracle's GEMM accumulates exactly for both FP8 variants
                    A, sa = oracle.quant_rows_fp8(x, q)
                    oracle.scaled_fp8_linear(A, sa, Wq, sw, bbits)
                else:
                    A, sa = oracle.quant_rows_int8(x, q)
                    oracle.scaled_int8_linear(A, sa, Wq, sw, bbits)
                t_total += time.perf_counter() - t0
                total_flops += 2 * x.shape[0] * lin.N * lin.K
                done.append(x.shape[0])
    desc = (f"{sum(done)} rows (per-token quantization + exact GEMM against the full per-channel "
            f"{dtype.upper()} weight) over the {len(wl.linears)} Linears of {wl.name}; "
            f"FLOPs of the sample / oracle time")
    return total_flops, t_total, desc


def _x_rows(wl, lin, n, seed):
    import numpy as np
    import torch
    from int8_w8a8_quantized_b200 import workloads
    r = wl.x_recipe
    x = workloads.activations(n, lin.K, seed=seed, nu=r.nu, amplitude=r.amplitude,
                              outlier_cols=int(round(r.outlier_frac * lin.K)), outlier_mult=r.outlier_mult)
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def cpu_baseline(wl, seconds, dtype="fp8", single_thread_seconds=None):
    """The oracle on every host core (OpenMP over rows), then on one core
    (a smaller sample of the same kind), both as FLOPs of the sample / time."""
    import oracle
    flops, secs, desc = oracle_sample(wl, seconds, dtype=dtype)
    out = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": desc, "seconds": secs}
    if single_thread_seconds:
        threads = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            f1, s1, d1 = oracle_sample(wl, single_thread_seconds, seed=1, dtype=dtype)
        finally:
            oracle.set_num_threads(threads)
        out["single_thread"] = {"value": f1 / s1 / 1e12, "unit": "TFLOP/s", "cores": 1, "sample": d1,
                                "seconds": s1}
    return out


# Dense 8-bit tensor-core rate of one B200 SM per clock (E4M3 or S8 operands):
# twice the 8192 bf16 FLOP/clk/SM behind the 2.25 PFLOP/s dense bf16 figure.
FP8_FLOP_PER_CLK_PER_SM = 16384


# Below this many milliseconds of timed region the sampled clock is not the
# clock the kernels ran at: the power limiter acts on a comparable time scale
# and the 10 ms sampler takes only a few samples.
SHORT_REGION_MS = 250.0


def clock_normalised(achieved_tflops, clocks, sm_count, region_ms=None):
    """The GEMM's rate against the tensor-core peak at the SM clock sampled
    during the timed region (SMs x 16384 FLOP/clk x median MHz): comparable
    between boxes whose power-capped clocks differ.  Flagged unreliable when
    the timed region is shorter than SHORT_REGION_MS."""
    mhz = (clocks or {}).get("sm_mhz")
    if not mhz or not sm_count:
        return None
    peak = sm_count * FP8_FLOP_PER_CLK_PER_SM * mhz * 1e6 / 1e12
    out = {"frac": round(achieved_tflops / peak, 4), "peak_at_clock": round(peak, 1), "sm_mhz": mhz,
           "sm_count": sm_count, "flop_per_clk_per_sm": FP8_FLOP_PER_CLK_PER_SM}
    if region_ms is not None and region_ms < SHORT_REGION_MS:
        out["reliable"] = False
        out["note"] = (f"timed region {region_ms:.0f} ms: too short for the sampled clock to be the clock the "
                       f"kernels ran at; run more --steps")
    return out


def path_roofline(res, steps, peaks, fp8_peak):
    """Floor of one step: every quantizer at the measured HBM copy bandwidth plus
    every GEMM at max(FLOPs / tensor peak, bytes / HBM bandwidth), against the
    measured step time; with the measured sustained 8-bit peak and with the
    4.5 PFLOP/s spec.  With launches that quantize inside the GEMM, also the
    floor of the overlapped step: such a launch at max(FLOPs / peak,
    (GEMM + quantizer bytes) / HBM)."""
    hbm = peaks.get("hbm_gbs", FALLBACK_HBM_GBS) * 1e9
    q_s = sum(res["step_quant_bytes"]) / hbm
    per_launch = list(zip(res["step_gemm_flops"], res["step_gemm_bytes"]))

    def floor_ms(peak_tflops):
        g_s = sum(max(f / (peak_tflops * 1e12), b / hbm) for f, b in per_launch)
        return 1e3 * (q_s + g_s)

    def overlapped_floor_ms(peak_tflops):
        return 1e3 * sum(max(f / (peak_tflops * 1e12), (g + q) / hbm) for _, f, g, q in res["step_ops"])

    measured = res["ms_per_step"]
    f_meas, f_spec = floor_ms(fp8_peak), floor_ms(FP8_SPEC_TFLOPS)
    out = {"floor_ms_measured_peaks": round(f_meas, 4), "frac_measured_peaks": round(f_meas / measured, 4),
           "floor_ms_spec": round(f_spec, 4), "frac_spec": round(f_spec / measured, 4),
           "model": "sum over quantizers of bytes / HBM + sum over GEMMs of max(FLOPs / peak, bytes / HBM)"}
    if any(kind == "fused" for kind, _, _, _ in res.get("step_ops", [])):
        o_meas, o_spec = overlapped_floor_ms(fp8_peak), overlapped_floor_ms(FP8_SPEC_TFLOPS)
        out["overlapped"] = {
            "floor_ms_measured_peaks": round(o_meas, 4), "frac_measured_peaks": round(o_meas / measured, 4),
            "floor_ms_spec": round(o_spec, 4), "frac_spec": round(o_spec / measured, 4),
            "model": "sum over launches of max(FLOPs / peak, bytes / HBM); a launch that quantizes inside its "
                     "GEMM moves its quantizer's bytes and its GEMM's"}
    return out


# ------------------------------------------------- quantizer-only workload
def quantizer_arm(args, rank, world, local_rank):
    """The activation-quantizer configuration: each step quantizes X [8192, 3072]
    per token to FP8 (qmax 448) and per row to INT8 (qmax 127).  X (48 MiB) fits
    in L2, so a 256 MiB buffer is written between timed steps and only the
    quantizer launches are timed (CUDA events around each step's two launches).
    The flush buffer is then read back, so that the dirty lines the write left
    in L2 are written back before the timed launches instead of during them."""
    import torch
    from int8_w8a8_quantized_b200 import _capi, workloads
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = _capi.load_library()
    stream = torch.cuda.current_stream()
    sh = int(stream.cuda_stream)
    x = workloads.quantizer_input(device=dev)
    M, K = x.shape
    q8 = torch.empty((M, K), dtype=torch.uint8, device=dev)
    s8 = torch.empty(M, device=dev)
    qi = torch.empty((M, K), dtype=torch.int8, device=dev)
    si = torch.empty(M, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {_capi.status_string(st)}: {_capi.last_error_message()}")

    def step():
        check(lib.tfq_quant_act_fp8_per_token(x.data_ptr(), M, K, 448.0, q8.data_ptr(), s8.data_ptr(), sh), "fp8")
        check(lib.tfq_quant_weight_per_channel(x.data_ptr(), M, K, _capi.TFQ_DTYPE_INT8, 127.0, qi.data_ptr(),
                                               si.data_ptr(), sh), "int8")

    sink = torch.empty(1, dtype=torch.int64, device=dev)
    flush_words = flush.view(torch.int64)

    def flush_l2():
        flush.zero_()
        torch.sum(flush_words, dim=0, keepdim=True, out=sink)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    evs = []
    for _ in range(args.steps):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True); e0.record(stream)
        step()
        e1 = torch.cuda.Event(enable_timing=True); e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    check(lib.tfq_device_error(sh), "device error")
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    nbytes = 2 * (3 * M * K + 4 * M)  # two quantizations: bf16 in, 8-bit codes + fp32 scale out
    # What this size allows: two device copies of the same traffic per step
    # (each reads and writes half of one launch's algorithmic bytes), timed
    # the same way.  Context for the fraction, not part of the metric.
    src = torch.empty(nbytes // 4, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    cevs = []
    for i in range(args.warmup + args.steps):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True); e0.record(stream)
        dst.copy_(src)
        dst.copy_(src)
        e1 = torch.cuda.Event(enable_timing=True); e1.record(stream)
        if i >= args.warmup:
            cevs.append((e0, e1))
    torch.cuda.synchronize()
    copy_ms = sum(a.elapsed_time(b) for a, b in cevs) / len(cevs)
    del src, dst
    value = world * nbytes / (ms * 1e-3) / 1e9
    peaks, peak_src = measured_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
    # end to end: X from pinned host memory, codes and scales back, every
    # step; H2D and D2H on two copy streams, so that the next step's input
    # crosses PCIe while this step's outputs go back.  The device input and
    # outputs are double-buffered (steps alternate between two sets), and
    # events keep each copy after the kernels that read or write its buffer.
    hx = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    hx.copy_(x)
    outs = [q8, s8, qi, si]
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    xbuf = [x, torch.empty_like(x)]
    obuf = [outs, [torch.empty_like(t) for t in outs]]
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    x_read, outs_read, counter = {}, {}, [0]

    def e2e_step():
        k = counter[0] % 2
        counter[0] += 1
        xk, (q8k, s8k, qik, sik) = xbuf[k], obuf[k]
        if k in x_read:
            copy_in.wait_event(x_read[k])
        with torch.cuda.stream(copy_in):
            xk.copy_(hx, non_blocking=True)
        landed = torch.cuda.Event()
        landed.record(copy_in)
        stream.wait_event(landed)
        if k in outs_read:
            stream.wait_event(outs_read[k])
        check(lib.tfq_quant_act_fp8_per_token(xk.data_ptr(), M, K, 448.0, q8k.data_ptr(), s8k.data_ptr(), sh),
              "fp8")
        check(lib.tfq_quant_weight_per_channel(xk.data_ptr(), M, K, _capi.TFQ_DTYPE_INT8, 127.0, qik.data_ptr(),
                                               sik.data_ptr(), sh), "int8")
        x_read[k] = torch.cuda.Event()
        x_read[k].record(stream)
        copy_out.wait_event(x_read[k])
        with torch.cuda.stream(copy_out):
            for h, t in zip(hout, obuf[k]):
                h.copy_(t, non_blocking=True)
        outs_read[k] = torch.cuda.Event()
        outs_read[k].record(copy_out)

    def copies_alone():
        copy_in.wait_stream(stream)
        copy_out.wait_stream(stream)
        with torch.cuda.stream(copy_in):
            x.copy_(hx, non_blocking=True)
        with torch.cuda.stream(copy_out):
            for h, t in zip(hout, outs):
                h.copy_(t, non_blocking=True)
        stream.wait_stream(copy_in)
        stream.wait_stream(copy_out)

    # a step is ~1 ms: enough steps that filling and draining the copy
    # pipeline are a small part of the timed region
    n_e2e = max(args.e2e_steps, 30)

    def timed(fn):
        fn()
        fn()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        copy_in.wait_stream(stream)  # no copy of the timed steps starts before t0
        copy_out.wait_stream(stream)
        for _ in range(n_e2e):
            fn()
        stream.wait_stream(copy_out)
        stream.wait_stream(copy_in)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n_e2e

    e2e_ms = timed(e2e_step)
    e2e_copy_ms = timed(copies_alone)
    if world > 1:  # the slowest rank times the job
        copy_ms = max_over_ranks(copy_ms, dev)
        e2e_ms = max_over_ranks(e2e_ms, dev)
        e2e_copy_ms = max_over_ranks(e2e_copy_ms, dev)
    if rank != 0:
        return
    line = {
        "metric": "activation quantizer GB/s (per-token FP8 qmax 448 + per-row INT8 127), algorithmic bytes",
        "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 + s8", "data": "synthetic",
        "config": {"workload": "activation_quantizer", "M": M, "K": K, "outlier_cols": "1 % x50",
                   "zero_rows": 16, "l2": "256 MiB written, then read, between timed steps (flush), not timed",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "quant_rows_kernel<fp8>, quant_rows_kernel<int8>", "bound": "hbm",
                     "achieved": round(value / world, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(value / world / hbm, 4), "frac_of_nominal_8tbs": round(value / world / 8000.0, 4),
                     "traffic": None, "algorithmic_bytes_per_launch": nbytes // 2, "peak_source": peak_src,
                     "same_traffic_copy": {"gbs": round(nbytes / (copy_ms * 1e-3) / 1e9, 1),
                                           "ms_per_step": round(copy_ms, 4),
                                           "frac": round(copy_ms / ms, 4),
                                           "what": "two device copies of the same bytes per step, same timing"}},
        "gpu_launches": 2 * args.steps, "clocks": clk,
        "e2e": {"value": round(world * nbytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": x.numel() * 2,
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs),
                "steps": n_e2e, "host_buffers": "pinned",
                "overlap": "H2D and D2H on two copy streams, overlapping the quantizers and each other; "
                           "device input and outputs double-buffered",
                "copies_alone_ms": round(e2e_copy_ms, 4), "frac_of_copy_floor": round(e2e_copy_ms / e2e_ms, 4),
                "floor": "the step's H2D and D2H copies alone, both directions at once, no kernels"},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = quantizer_cpu_baseline(x.cpu(), args.cpu_seconds,
                                                      single_thread_seconds=max(2.0, args.cpu_seconds / 2))
    print(json.dumps(line), flush=True)


def quantizer_cpu_baseline(x_cpu, seconds: float = 10.0, single_thread_seconds=None):
    """The oracle's FP8 and INT8 quantizers over the whole input, on every
    host core; then (optionally) on one core."""
    import numpy as np
    import torch
    import oracle
    bits = x_cpu.contiguous().view(torch.int16).numpy().view(np.uint16)
    M, K = bits.shape

    def passes(limit):
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < limit or n == 0:
            oracle.quant_rows_fp8(bits, 448.0)
            oracle.quant_rows_int8(bits, 127.0)
            n += 1
        return n, time.perf_counter() - t0

    n, secs = passes(seconds)
    out = {"value": n * 2 * (3 * M * K + 4 * M) / secs / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
           "kind": "oracle", "sample": f"{n} passes over the full [{M}, {K}] input (FP8 and INT8)", "seconds": secs,
           "ms_per_pass": 1e3 * secs / n}
    if single_thread_seconds:
        threads = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            n1, s1 = passes(single_thread_seconds)
        finally:
            oracle.set_num_threads(threads)
        out["single_thread"] = {"value": n1 * 2 * (3 * M * K + 4 * M) / s1 / 1e9, "unit": "GB/s", "cores": 1,
                                "sample": f"{n1} passes over the full [{M}, {K}] input (FP8 and INT8)",
                                "seconds": s1}
    return out


def use_all_host_cores_for_oracle():
    """The reference arm runs on rank 0 alone (the other ranks exit without
    work), so the oracle gets every core this process may use, as in a plain
    N = 1 run -- torchrun sets OMP_NUM_THREADS=1 for each rank otherwise."""
    import oracle
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    oracle.set_num_threads(max(1, n))


# ------------------------------------------------------------------ main
def quantizer_main(args, rank, world, local_rank):
    if args.impl == "reference":
        if rank != 0:
            return 0
        from int8_w8a8_quantized_b200 import workloads
        import oracle
        use_all_host_cores_for_oracle()
        x = workloads.quantizer_input()
        cb = quantizer_cpu_baseline(x, args.cpu_seconds)
        line = {"metric": "activation quantizer GB/s (per-token FP8 qmax 448 + per-row INT8 127), algorithmic bytes",
                "impl": "reference", "value": cb["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": cb["ms_per_pass"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": "activation_quantizer", "M": 8192, "K": 3072},
                "cpu_baseline": {"value": cb["value"], "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": cb["sample"]},
                "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    quantizer_arm(args, rank, world, local_rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from int8_w8a8_quantized_b200 import workloads
    if args.workload == "activation_quantizer":
        return quantizer_main(args, rank, world, local_rank)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses
        wl = dataclasses.replace(wl, M=args.tokens)
    if args.fused and args.dtype != "fp8":
        raise SystemExit("--fused takes --dtype fp8")
    # FP8 and INT8 without --fused: the Linears that share an activation as one launch
    args.multi = args.dtype in ("fp8", "int8") and not args.fused and not args.separate
    cfg = {"workload": wl.name, "M": wl.M, "dtype": args.dtype,
           "linears": [f"{l.name}:{l.K}->{l.N}" for l in wl.linears],
           "act_qmax": list(act_qmaxes(wl, args.dtype)) if args.dtype != "mxfp8" else "none (E8M0 scale per 32 values)",
           "weight_qmax": 448.0 if args.dtype != "mxfp8" else "none (E8M0 scale per 32 values)",
           "bias": wl.has_bias,
           "l2": l2_note(wl),
           "parallelism": f"replicas x{world}"}
    if args.fused:
        cfg["quantization"] = "inside the first GEMM of each activation (one kernel per Linear)"
    if args.multi:
        cfg["launches"] = "the Linears that read one activation (Q, K, V) as one GEMM launch"
    if args.tokens:
        cfg["reduced_tokens"] = f"M = {args.tokens} instead of the workload's M (a profiling case, not a benchmark)"

    if args.impl == "reference":
        if rank != 0:
            return 0
        use_all_host_cores_for_oracle()
        reference_arm(args, wl, cfg, world)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res, e2e = gpu_arm(args, wl, rank, world, local_rank)
    if world > 1:
        if e2e is not None:  # every rank measured its own replica; the slowest one times the job
            slowest = max_over_ranks(e2e["ms_per_step"], torch.device("cuda", local_rank))
            e2e["value"] *= e2e["ms_per_step"] / slowest
            e2e["ms_per_step"] = slowest
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = measured_peaks()
    flops_step = wl.flops() // len(wl.act_qmax) * len(act_qmaxes(wl, args.dtype))
    value = aggregate_throughput(world, flops_step, res["ms_per_step"])
    fused = res["fused_launches"] > 0
    if fused:  # the dominant kernel is the GEMM that quantizes its own activations
        gemm_avg_ms = res["fused_ms_total"] / res["fused_launches"]
        gemm_tflops = res["fused_flops_total"] / (res["fused_ms_total"] * 1e-3) / 1e12
        gemm_alg_bytes = round(res["fused_bytes_total"] / res["fused_launches"])
    else:
        gemm_avg_ms = res["gemm_ms_total"] / max(1, res["gemm_launches"])
        gemm_tflops = res["gemm_flops_total"] / (res["gemm_ms_total"] * 1e-3) / 1e12
        gemm_alg_bytes = round(res["gemm_bytes_total"] / max(1, res["gemm_launches"]))
    # The GEMMs run back to back for the whole timed region (the power cap
    # holds the clocks down within ~0.1 s), so the sustained measured peak
    # is the denominator; the burst fraction is reported beside it.
    bf16_sus = peaks.get("bf16_tflops_sustained", 1400.0)
    bf16_burst = peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)
    fp8_peak = bf16_sus * FP8_OVER_BF16
    pair = wl.M >= 512
    if args.dtype == "mxfp8":
        kname = "mxfp8_mm_pair_kernel" if pair else "mxfp8_mm_kernel"
        qname = "quant_mxfp8_blocks_kernel"
    else:
        kname = ("scaled_mm_pair_kernel" if pair else "scaled_mm_kernel") + f"<{args.dtype}>"
        qname = "quant_rows_kernel<" + args.dtype + ">"
        if fused:
            kname = "scaled_mm_pair_kernel<fp8, quantizing its activations>"
    quant_gbs = res["quant_bytes_total"] / (res["quant_ms_total"] * 1e-3) / 1e9 if res["quant_ms_total"] else None
    line = {
        "metric": metric_name(args.dtype),
        "value": round(value, 2),
        "unit": unit_name(args.dtype),
        "pct_fp8_dense_peak": round(100.0 * value / (world * FP8_SPEC_TFLOPS), 2),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(res["ms_per_step"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"fp8": "e4m3", "int8": "s8", "fp8_f16acc": "e4m3 (f16 accumulate)",
                  "mxfp8": "e4m3 (e8m0 block-32 scales)"}[args.dtype],
        "data": "synthetic",
        "config": cfg,
        "roofline": {
            "kernel": kname,
            "bound": "tensor",
            "achieved": round(gemm_tflops, 1),
            "peak": round(fp8_peak, 1),
            "unit": unit_name(args.dtype),
            "frac": round(gemm_tflops / fp8_peak, 4),
            "traffic": None if fused else recorded_traffic("gemm", wl.name, args.dtype),
            "algorithmic_bytes_per_launch": gemm_alg_bytes,
            "peak_source": f"{peak_src} bf16 sustained x {FP8_OVER_BF16} (nominal fp8|int8 / bf16 dense ratio)",
            "frac_of_burst_peak": round(gemm_tflops / (bf16_burst * FP8_OVER_BF16), 4),
            "avg_launch_ms": round(gemm_avg_ms, 4),
            "frac_of_fp8_spec": round(gemm_tflops / FP8_SPEC_TFLOPS, 4),
            "clock_normalised": clock_normalised(gemm_tflops, res["clocks"], res.get("sm_count"),
                                                 res["ms_per_step"] * args.steps),
        },
        "quantizer": {"inside": "the fused launches quantize their activations (quantizer warps of the GEMM "
                                "kernel); no quantizer launch of its own"} if fused else {
            "kernel": qname,
            "bound": "hbm",
            "achieved": None if quant_gbs is None else round(quant_gbs, 1),
            "peak": peaks.get("hbm_gbs", FALLBACK_HBM_GBS),
            "unit": "GB/s",
            "frac": None if quant_gbs is None else round(quant_gbs / peaks.get("hbm_gbs", FALLBACK_HBM_GBS), 4),
            "frac_of_nominal_8tbs": None if quant_gbs is None else round(quant_gbs / 8000.0, 4),
            "share_of_step": round(res["quant_ms_total"] / max(1, res["quant_launches"]) *
                                   res["quant_launches_per_step"] / res["ms_per_step"], 4),
            "traffic": recorded_traffic("quant", wl.name, args.dtype),
            "algorithmic_bytes_per_launch": round(res["quant_bytes_total"] / max(1, res["quant_launches"])),
            "in_step_copy": None if not res.get("quant_copy_reference") or quant_gbs is None else dict(
                res["quant_copy_reference"], gbs=round(res["quant_copy_reference"]["gbs"], 1),
                frac=round(quant_gbs / res["quant_copy_reference"]["gbs"], 4)),
        },
        "path_roofline": path_roofline(res, args.steps, peaks, fp8_peak),
        "context": res.get("context"),
        "per_linear_ms": {k: round(statistics.median(v), 4) for k, v in res["per_linear"].items()},
        "gpu_launches": res["gpu_launches"],
        "kernel_events": res["kernel_events"],
        "nonfinite_outputs": res["nonfinite_outputs"],
        "clocks": res["clocks"],
    }
    if e2e is not None:
        e2e["value"] = round(world * e2e["value"], 3)
        line["e2e"] = e2e
    clk = res["clocks"] or {}
    if clk.get("power_w_instant_median") and value > 0:
        line["energy"] = {"pj_per_op": round(clk["power_w_instant_median"] / (value / world), 4),
                          "what": "median instantaneous board power in the timed region / this GPU's rate "
                                  "(W per TFLOP/s = pJ per FLOP or OP, quantizers included)"}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, args.dtype,
                                            single_thread_seconds=max(2.0, args.cpu_seconds / 2))
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args, wl, cfg, world):
    """The oracle, as it stands, timed on the host cores; each step is a
    bounded sample of the workload."""
    import oracle
    per_step = max(2.0, min(15.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(wl, per_step, seed=1000 + i, dtype=args.dtype)
    flops = 0
    secs = 0.0
    desc = ""
    for i in range(args.steps):
        f, s, desc = oracle_sample(wl, per_step, seed=i, dtype=args.dtype)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "metric": metric_name(args.dtype), "impl": "reference", "value": value, "unit": unit_name(args.dtype),
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": unit_name(args.dtype), "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": unit_name(args.dtype), "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    sys.exit(main())
