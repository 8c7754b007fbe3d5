"""The allocation-free GEMM entry point (tfq_scaled_fp8_linear_noalloc).

It serves callers that must not allocate device memory (a framework that
owns all device memory through its own pool, a process that reserved most of
HBM, code where a possibly synchronizing CUDA call is not allowed): its only
scratch, the word a kernel writes when a bounded wait runs out, lives in a
static device array instead of a cudaMalloc'd buffer.  This test calls it
through the C ABI twice in a row (different shapes, so the second call runs
on the array the first one left behind) and checks each output against the
regular entry point's output within the GEMM tolerance the other tests use.
It lives in a file that pytest collects last and passes both alone in a
fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from int8_w8a8_quantized_b200 import _capi
from tests import _gpu

pytestmark = pytest.mark.gpu


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


def test_noalloc_matches_regular_entry_point_twice():
    lib = _gpu.lib()
    for M, N, K, seed, with_bias in [(300, 520, 1024, 1, True), (129, 264, 144, 2, False)]:
        A, sa, W, sw, b = _inputs(M, N, K, seed, with_bias)
        y_noalloc = _call(lib.tfq_scaled_fp8_linear_noalloc, A, sa, W, sw, b)
        y_regular = _call(lib.tfq_scaled_fp8_linear, A, sa, W, sw, b)
        _gpu.gemm_tolerance_check(y_noalloc, y_regular.double().cpu().numpy(), f"noalloc M={M} N={N} K={K}")
