"""The allocation-free GEMM entry point (tfq_scaled_fp8_linear_noalloc).

It serves callers that must not allocate device memory: a framework that
owns all device memory through its own pool, or a process that reserved
most of HBM up front.  The regular entry points cudaMalloc a small per-device
buffer on their first call; this one keeps the same words (the error word a
kernel writes when a bounded wait runs out, and the counters the CTA-pair
kernel's clusters keep pace with) in a static device array instead.

The tests call it through the C ABI, two calls in a row per shape, on shapes
that run the one-CTA kernel (M < 512) and the CTA-pair kernel with several
rounds of tiles per cluster (so the pacing counters in the static array are
used, and the second call runs on the array the first one left behind).
Each output is checked against the oracle and against the regular entry
point's output, within the GEMM tolerance the other tests use.  A second test
checks, in a fresh process, that repeated calls leave the device's free
memory unchanged.  This file is collected last and passes both alone in a
fresh process and after the other tests.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi
from tests import _gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (M, N, K, seed, bias): one-CTA kernel; CTA pairs, one round; CTA pairs,
# 192 tiles over 74 clusters (three rounds, pacing counters in use).
SHAPES = [(300, 520, 1024, 1, True), (129, 264, 144, 2, False), (2128, 1032, 512, 3, True),
          (4096, 3072, 1024, 4, True)]


def _inputs(M, N, K, seed, with_bias):
    g = torch.Generator().manual_seed(seed)
    mag = torch.randint(0, 0x70, (M, K), generator=g, dtype=torch.int32)
    A = (mag | (torch.randint(0, 2, (M, K), generator=g, dtype=torch.int32) << 7)).to(torch.uint8)
    mag = torch.randint(0, 0x70, (N, K), generator=g, dtype=torch.int32)
    W = (mag | (torch.randint(0, 2, (N, K), generator=g, dtype=torch.int32) << 7)).to(torch.uint8)
    sa = torch.rand(M, generator=g) * 0.01 + 1e-4
    sw = torch.rand(N, generator=g) * 0.01 + 1e-4
    b = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if with_bias else None
    return [t if t is None else t.cuda() for t in (A, sa, W, sw, b)]


def _call(fn, A, sa, W, sw, b):
    M, K = A.shape
    N = W.shape[0]
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    st = fn(A.data_ptr(), sa.data_ptr(), W.data_ptr(), sw.data_ptr(), None if b is None else b.data_ptr(),
            M, N, K, out.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, (_capi.status_string(st), _capi.last_error_message())
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("M,N,K,seed,with_bias", SHAPES)
def test_noalloc_matches_oracle_and_regular_entry_point_twice(M, N, K, seed, with_bias):
    lib = _gpu.lib()
    A, sa, W, sw, b = _inputs(M, N, K, seed, with_bias)
    y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), W.cpu().numpy(), sw.cpu().numpy(),
                                     None if b is None else _gpu.bf16_bits_np(b))
    y_regular = _call(lib.tfq_scaled_fp8_linear, A, sa, W, sw, b)
    for call in range(2):
        y = _call(lib.tfq_scaled_fp8_linear_noalloc, A, sa, W, sw, b)
        what = f"noalloc call {call} M={M} N={N} K={K}"
        _gpu.gemm_tolerance_check(y, y_ref, what + " vs oracle")
        _gpu.gemm_tolerance_check(y, y_regular.double().cpu().numpy(), what + " vs regular entry point")


_NO_ALLOC_SCRIPT = textwrap.dedent("""
    import json, torch
    from int8_w8a8_quantized_b200 import _capi
    lib = _capi.load_library()
    torch.cuda.init()
    shapes = [(300, 520, 1024), (2128, 1032, 512), (4096, 3072, 1024)]
    bufs = []
    for M, N, K in shapes:  # every buffer exists before the first measurement
        A = torch.randint(0, 0x70, (M, K), dtype=torch.uint8, device="cuda")
        W = torch.randint(0, 0x70, (N, K), dtype=torch.uint8, device="cuda")
        sa = torch.full((M,), 1e-3, device="cuda")
        sw = torch.full((N,), 1e-3, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        bufs.append((A, sa, W, sw, out, M, N, K))
    stream = int(torch.cuda.current_stream().cuda_stream)

    def calls():
        for A, sa, W, sw, out, M, N, K in bufs:
            st = lib.tfq_scaled_fp8_linear_noalloc(A.data_ptr(), sa.data_ptr(), W.data_ptr(), sw.data_ptr(),
                                                   None, M, N, K, out.data_ptr(), stream)
            assert st == 0, _capi.last_error_message()
        torch.cuda.synchronize()

    calls()  # first calls: one-time set-up, the runtime loads the kernels' code
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        calls()
    free1 = torch.cuda.mem_get_info()[0]
    print(json.dumps({"free_before": free0, "free_after": free1}))
""")


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """In a fresh process that never calls a regular entry point: after the
    first calls (the one-time set-up, and the runtime loading the kernels'
    code), three more rounds of calls on three shapes leave the device's free
    memory, as the driver reports it, unchanged."""
    r = subprocess.run([sys.executable, "-c", _NO_ALLOC_SCRIPT], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    import json
    info = json.loads(r.stdout.strip().splitlines()[-1])
    assert info["free_after"] == info["free_before"], info
