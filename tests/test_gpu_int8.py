"""GPU parity of the INT8 W8A8 path (NEXT row f2): per-token INT8 activation
codes bit-exact with the oracle, the S8 x S8 -> S32 tensor-core GEMM with the
fused epilogue within |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref) of the
oracle's exact integer sums."""
import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi, workloads
from tests import _gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _gpu.lib()


def _int8_linear(A, sa, W, sw, b):
    M, K = A.shape
    N = W.shape[0]
    out = _gpu.guarded(M * N, torch.bfloat16, 12345.0)
    st = _capi.raw.tfq_scaled_int8_linear(A.data_ptr(), sa.data_ptr(), W.data_ptr(), sw.data_ptr(),
                                          None if b is None else b.data_ptr(), M, N, K, out.data_ptr(),
                                          _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    assert torch.all(out[M * N:] == 12345.0), "write past the end of the output"
    return out[:M * N].view(M, N)


def _quant_act_int8(x, qmax=127.0):
    M, K = x.shape
    q = _gpu.guarded(M * K, torch.int8, 99)
    s = _gpu.guarded(M, torch.float32, -7.0)
    st = _capi.raw.tfq_quant_act_int8_per_token(x.data_ptr(), M, K, float(qmax), q.data_ptr(), s.data_ptr(),
                                                _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    assert torch.all(q[M * K:] == 99) and torch.all(s[M:] == -7.0)
    return q[:M * K].view(M, K), s[:M]


def _case(M, N, K, with_bias, seed, lo=-128, hi=128):
    g = torch.Generator().manual_seed(seed)
    A = torch.randint(lo, hi, (M, K), generator=g, dtype=torch.int8)
    W = torch.randint(lo, hi, (N, K), generator=g, dtype=torch.int8)
    sa = torch.rand(M, generator=g) * 1e-3 + 1e-5
    sw = torch.rand(N, generator=g) * 1e-3 + 1e-5
    b = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if with_bias else None
    y = _int8_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None if b is None else b.cuda())
    y_ref = oracle.scaled_int8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(),
                                      None if b is None else _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, f"int8 M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (100, 136, 48), (129, 264, 144), (300, 520, 1024),
                                   (512, 256, 128), (777, 520, 1024), (2128, 1032, 512)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_int8_ragged_full_compare(M, N, K, with_bias):
    _case(M, N, K, with_bias, seed=M * 3 + N + K)


def test_int8_extreme_codes():
    """All codes at -128/127 with K = 13824: |sum| up to 2.3e8 stays exact in s32."""
    M, N, K = 600, 264, 13824
    A = torch.full((M, K), 127, dtype=torch.int8)
    A[::2, ::3] = -128
    W = torch.full((N, K), -128, dtype=torch.int8)
    W[1::2, 1::5] = 127
    sa = torch.full((M,), 1e-4)
    sw = torch.full((N,), 2e-4)
    y = _int8_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None)
    y_ref = oracle.scaled_int8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy())
    _gpu.gemm_tolerance_check(y, y_ref, "int8 extreme")


@pytest.mark.parametrize("M,N", [(3, 8), (512, 136)])
def test_int8_sum_at_the_largest_k(M, N):
    """K = TFQ_INT8_MAX_K - 16, the largest K the INT8 GEMM takes, with every
    product at 128^2: |sum| = 16384 K = 2 147 221 504, just below 2^31, so
    the s32 accumulator is still exact (one-CTA and CTA-pair kernels)."""
    K = _capi.TFQ_INT8_MAX_K - 16
    A = torch.full((M, K), -128, dtype=torch.int8)
    W = torch.full((N, K), -128, dtype=torch.int8)
    W[1::2] = 127                                   # rows of -128 * 127 products: sums of the other sign
    sa = torch.full((M,), 1e-6)
    sw = torch.full((N,), 2e-6)
    y = _int8_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None)
    y_ref = oracle.scaled_int8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy())
    assert y_ref[0, 0] == 16384.0 * K * float(np.float32(1e-6)) * float(np.float32(2e-6))
    _gpu.gemm_tolerance_check(y, y_ref, f"int8 K={K}")


def test_int8_linear_end_to_end():
    x = workloads.activations(700, 1024, seed=21, nu=4, outlier_cols=10, outlier_mult=20.0, zero_rows=3,
                              device="cuda")
    w = workloads.weights(520, 1024, seed=22, std=0.02, device="cuda")
    b = workloads.bias(520, seed=23, device="cuda")
    A, sa = _quant_act_int8(x)
    A_ref, sa_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(A.cpu().numpy(), A_ref)
    np.testing.assert_array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_INT8, 127.0)
    W_ref, sw_ref = _gpu.oracle_quant_int8(w, 127.0)
    np.testing.assert_array_equal(Wq.cpu().numpy().view(np.int8), W_ref)
    y = _int8_linear(A, sa, Wq.view(torch.int8), sw, b)
    y_ref = oracle.scaled_int8_linear(A_ref, sa_ref, W_ref, sw_ref, _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "int8 end to end")


def test_int8_full_size_sampled():
    """Video-DiT FFN-down at full size (75600 x 13824 -> 5120) through the
    INT8 path; one row of every 128-row CTA share of every M tile, 512 more
    seeded rows and the ragged tail, all N columns."""
    wl = workloads.VIDEO_DIT
    lin = [l for l in wl.linears if l.name == "ffn_down"][0]
    x = wl.make_x(lin.x, device="cuda")
    w = wl.make_w(lin, device="cuda")
    b = wl.make_bias(lin, device="cuda")
    A, sa = _quant_act_int8(x)
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_INT8, 127.0)
    y = _int8_linear(A, sa, Wq.view(torch.int8), sw, b)
    rows = _gpu.tile_sample_rows(wl.M, seed=5)
    A_ref, sa_ref = _gpu.oracle_quant_int8(x, 127.0, rows)
    np.testing.assert_array_equal(A[torch.as_tensor(rows, device="cuda")].cpu().numpy(), A_ref)
    y_ref = oracle.scaled_int8_linear(A.cpu().numpy(), sa.cpu().numpy(), Wq.view(torch.int8).cpu().numpy(),
                                      sw.cpu().numpy(), _gpu.bf16_bits_np(b), rows=rows)
    _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, "int8 video ffn_down")


def test_int8_tensor_wrappers():
    from int8_w8a8_quantized_b200 import tfq_quant_weight_per_channel, w8a8_int8_linear
    x = workloads.activations(300, 512, seed=9, device="cuda")
    w = workloads.weights(264, 512, seed=10, std=0.02, device="cuda")
    Wq, sw = tfq_quant_weight_per_channel(w, "int8")
    y = w8a8_int8_linear(x, Wq, sw, None)
    A_ref, sa_ref = _gpu.oracle_quant_int8(x, 127.0)
    y_ref = oracle.scaled_int8_linear(A_ref, sa_ref, Wq.cpu().numpy(), sw.cpu().numpy(), None)
    _gpu.gemm_tolerance_check(y, y_ref, "int8 wrapper")


@pytest.mark.parametrize("K", [528, 5120, 16384])
def test_int8_rounding_edges(K):
    """INT8 codes where x/s is an exact half-integer (round half to even
    decides), signed zeros, values that round to 0, rows below the 1e-12
    floor and rows whose scale exceeds 2^64 (the IEEE-division branch), for
    the grouped, one-warp-per-row and shared-memory-staged kernels."""
    halves = torch.arange(-127, 127, dtype=torch.float32) + 0.5
    row = torch.cat([torch.tensor([127.0, -127.0]), halves, torch.tensor([-0.0, 0.0, 0.25, -0.25, 0.75, 1e-30])])
    reps = (K + row.numel() - 1) // row.numel()
    base = row.repeat(reps)[:K]
    x = torch.zeros(8, K)
    x[0] = base                        # s = 1: x/s = x exactly
    x[1] = base * 2.0 ** -20           # s = 2^-20, same quotients
    x[2] = base * 2.0 ** 100           # s = 2^100
    x[3] = -0.0
    x[4, :4] = torch.tensor([1e-13, -3e-13, 2e-13, -1e-14])   # below the floor
    x[5] = base * 3.0                  # a scale that is not a power of two
    x[6] = base * (3.0e38 / 127.0)     # s > 2^64 for every qmax
    x[7] = -base
    x = x.to(torch.bfloat16).cuda()
    assert torch.isfinite(x.float()).all()
    for qmax in (127.0, 100.0, 63.5, 2.0, 1.0):
        q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, qmax)
        q_ref, s_ref = _gpu.oracle_quant_int8(x, qmax)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


@pytest.mark.parametrize("M,N,K", [(2523, 1992, 256), (4096, 4096, 128)])
def test_int8_split_last_round(M, N, K):
    """The INT8 pair kernel with its last round split into half-width tiles."""
    _case(M, N, K, True, seed=M + 5 * N + K)


@pytest.mark.parametrize("M,N,K", [(9400, 1000, 400), (18944, 1536, 128)])
def test_int8_pair_kernel_large(M, N, K):
    """The INT8 pair kernel on a ragged 148-tile shape and a 444-tile one (six rounds)."""
    _case(M, N, K, True, seed=M + 3 * N + K)
