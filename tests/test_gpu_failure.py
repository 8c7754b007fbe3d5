"""Failure detection on the GPU without a fault: a kernel whose wait can only
run out (a barrier nothing completes) gives up after a short limit through
the same bounded-wait helper the GEMM roles use, records it in the device
error word and returns.  tfq_device_error() reports TFQ_ETIMEOUT once, then
the word is clear and the context still computes correct results."""
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi
from tests import _gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    lib = _gpu.lib()
    sh = _gpu.stream_handle()
    assert lib.tfq_device_error(sh) == _capi.TFQ_OK            # clean start
    assert lib.tfq_selftest_wait_timeout(20000, sh) == _capi.TFQ_OK   # 20 ms limit
    st = lib.tfq_device_error(sh)
    assert st == _capi.TFQ_ETIMEOUT, _capi.status_string(st)
    assert "bounded device wait" in _capi.last_error_message()
    assert lib.tfq_device_error(sh) == _capi.TFQ_OK            # cleared
    # the context is still usable: a GEMM afterwards is correct
    g = torch.Generator().manual_seed(0)
    A = torch.randint(0, 0x70, (300, 256), generator=g, dtype=torch.int32).to(torch.uint8)
    W = torch.randint(0, 0x70, (136, 256), generator=g, dtype=torch.int32).to(torch.uint8)
    sa = torch.rand(300, generator=g) * 1e-2
    sw = torch.rand(136, generator=g) * 1e-2
    y = _gpu.scaled_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None)
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy())
    _gpu.gemm_tolerance_check(y, y_ref, "after timeout")


def test_selftest_rejects_bad_limits():
    lib = _gpu.lib()
    assert lib.tfq_selftest_wait_timeout(0, _gpu.stream_handle()) == _capi.TFQ_EINVAL
    assert lib.tfq_selftest_wait_timeout(10000001, _gpu.stream_handle()) == _capi.TFQ_EINVAL
