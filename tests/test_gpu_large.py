"""Problems past 2^31 elements: the quantizers' and the GEMM's 64-bit
offsets (row * K, block index * 64 bytes, row * N) at sizes where a 32-bit
offset would wrap.  Each input is a few GB on the device; the oracle checks
a seeded sample of rows plus the rows around the first 2^31-element offset
and the last rows, codes and scales bit-exact, the GEMM within the stated
tolerance."""
import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi
from tests import _gpu

pytestmark = pytest.mark.gpu

LIMIT = 2 ** 31


def _rows(M, K, seed):
    r = _gpu.sample_rows(M, 48, seed)
    edge = LIMIT // K
    return np.unique(np.concatenate([r, np.arange(max(0, edge - 2), min(M, edge + 3))])).astype(np.int64)


def _big_x(M, K, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    x.normal_(generator=g)
    x[:, :: max(1, K // 31)] *= 30.0   # outlier columns
    x[7::1009] = 0.0                   # some all-zero rows
    return x


@pytest.mark.parametrize("M,K", [(1_100_000, 2048), (160_000, 13824), (140_000, 16384)])
def test_row_quantizers_past_2p31_elements(M, K):
    """The grouped (K = 2048), one-warp-per-row (K = 13824) and shared-memory
    staged (K = 16384) row quantizers, FP8 and INT8."""
    assert M * K > LIMIT
    x = _big_x(M, K, seed=K)
    rows = _rows(M, K, seed=K + 1)
    ridx = torch.as_tensor(rows, device="cuda")
    st = _gpu.stream_handle()
    q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    assert _capi.raw.tfq_quant_act_fp8_per_token(x.data_ptr(), M, K, 448.0, q.data_ptr(), s.data_ptr(), st) == 0
    _gpu.check_device_error()
    q_ref, s_ref = _gpu.oracle_quant_fp8(x, 448.0, rows)
    np.testing.assert_array_equal(s[ridx].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q[ridx].cpu().numpy(), q_ref)
    assert _capi.raw.tfq_quant_weight_per_channel(x.data_ptr(), M, K, _capi.TFQ_DTYPE_INT8, 127.0, q.data_ptr(),
                                                  s.data_ptr(), st) == 0
    _gpu.check_device_error()
    qi_ref, si_ref = _gpu.oracle_quant_int8(x, 127.0, rows)
    np.testing.assert_array_equal(s[ridx].cpu().numpy().view(np.uint32), si_ref.view(np.uint32))
    np.testing.assert_array_equal(q[ridx].cpu().numpy().view(np.int8), qi_ref)
    del x, q, s
    torch.cuda.empty_cache()


def test_mxfp8_quantizer_past_2p31_elements():
    """The MXFP8 quantizer's flat block index (block * 64 bytes) past 2^31 bytes
    and elements; scale codes read back from the tensor-core layout."""
    M, K = 70_000, 32768
    assert M * K > LIMIT
    x = _big_x(M, K, seed=3)
    rows = _rows(M, K, seed=4)
    nb = int(_capi.raw.tfq_mxfp8_scale_bytes(M, K))
    q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sf = torch.empty((nb,), dtype=torch.uint8, device="cuda")
    assert _capi.raw.tfq_quant_mxfp8(x.data_ptr(), M, K, q.data_ptr(), sf.data_ptr(), _gpu.stream_handle()) == 0
    _gpu.check_device_error()
    q_ref, sf_ref = oracle.quant_mxfp8(_gpu.bf16_bits_np(x[torch.as_tensor(rows, device="cuda")]))
    ridx = torch.as_tensor(rows, device="cuda")
    np.testing.assert_array_equal(q[ridx].cpu().numpy(), q_ref)
    ra = (M + 127) // 128
    b = np.arange(K // 32, dtype=np.int64)[None, :]
    r = rows[:, None]
    off = ((b // 4) * ra + r // 128) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    np.testing.assert_array_equal(sf.cpu().numpy()[off], sf_ref)
    del x, q, sf
    torch.cuda.empty_cache()


def test_gemm_past_2p31_outputs():
    """A GEMM with more than 2^31 output elements (row * N past 2^31): the
    epilogue's stores, the row scales and the raster at M = 160000."""
    M, N, K = 160_000, 16384, 256
    assert M * N > LIMIT
    g = torch.Generator().manual_seed(9)
    mag = torch.randint(0, 0x70, (M, K), generator=g, dtype=torch.int32)
    A = (mag | (torch.randint(0, 2, (M, K), generator=g, dtype=torch.int32) << 7)).to(torch.uint8)
    mag = torch.randint(0, 0x70, (N, K), generator=g, dtype=torch.int32)
    W = (mag | (torch.randint(0, 2, (N, K), generator=g, dtype=torch.int32) << 7)).to(torch.uint8)
    sa = torch.rand(M, generator=g) * 1e-2 + 1e-4
    sw = torch.rand(N, generator=g) * 1e-2 + 1e-4
    b = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Ad, Wd, sad, swd, bd = A.cuda(), W.cuda(), sa.cuda(), sw.cuda(), b.cuda()
    assert _capi.raw.tfq_scaled_fp8_linear(Ad.data_ptr(), sad.data_ptr(), Wd.data_ptr(), swd.data_ptr(),
                                           bd.data_ptr(), M, N, K, y.data_ptr(), _gpu.stream_handle()) == 0
    _gpu.check_device_error()
    rows = _rows(M, N, seed=10)
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(), _gpu.bf16_bits_np(b), rows=rows)
    _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, "M*N > 2^31")
    del y, Ad, Wd
    torch.cuda.empty_cache()
