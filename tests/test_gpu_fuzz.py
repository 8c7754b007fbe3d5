"""Seeded random shapes through every kernel, full comparison with the
oracle: sizes drawn across the kernels' dispatch boundaries (grouped,
one-warp-per-row and staged quantizers; one-CTA and CTA-pair GEMMs, split
last rounds, M, N and K tails), qmax drawn from the values the pages use and
two that exercise the clamp.  Codes and scales bit-exact, GEMMs within the
stated tolerance."""
import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi, workloads
from tests import _gpu
from tests.test_gpu_mxfp8 import _check_quant as _check_mx_quant

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(20261202)
QUANT_SHAPES = [(int(RNG.integers(1, 3000)), int(RNG.integers(1, 1400)) * 16) for _ in range(24)]
GEMM_SHAPES = []
while len(GEMM_SHAPES) < 20:
    M, N, K = int(RNG.integers(1, 2600)), int(RNG.integers(1, 300)) * 8, int(RNG.integers(1, 200)) * 16
    if M * N * K <= 3 * 2 ** 31:
        GEMM_SHAPES.append((M, N, K))
MX_SHAPES = [(int(RNG.integers(1, 1800)), int(RNG.integers(1, 160)) * 8, int(RNG.integers(1, 96)) * 32)
             for _ in range(12)]
QMAXES = [448.0, 14.0, 7.0, 21.0, 100.0]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _gpu.lib()


@pytest.mark.parametrize("i", range(len(QUANT_SHAPES)))
def test_row_quantizers(i):
    M, K = QUANT_SHAPES[i]
    qmax = QMAXES[i % len(QMAXES)]
    x = workloads.activations(M, K, seed=1000 + i, nu=3 + i % 3, outlier_cols=1 + i % 5, outlier_mult=25.0,
                              zero_rows=1 if M > 3 else 0, device="cuda")
    q, s = _gpu.quant_act_fp8(x, qmax)
    q_ref, s_ref = _gpu.oracle_quant_fp8(x, qmax)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    qi, si = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0 if i % 2 else 63.5)
    qi_ref, si_ref = _gpu.oracle_quant_int8(x, 127.0 if i % 2 else 63.5)
    np.testing.assert_array_equal(si.cpu().numpy().view(np.uint32), si_ref.view(np.uint32))
    np.testing.assert_array_equal(qi.cpu().numpy().view(np.int8), qi_ref)


def _codes(g, shape):
    mag = torch.randint(0, 0x70, shape, generator=g, dtype=torch.int32)
    return (mag | (torch.randint(0, 2, shape, generator=g, dtype=torch.int32) << 7)).to(torch.uint8)


@pytest.mark.parametrize("i", range(len(GEMM_SHAPES)))
def test_fp8_and_int8_gemms(i):
    M, N, K = GEMM_SHAPES[i]
    g = torch.Generator().manual_seed(2000 + i)
    A, W = _codes(g, (M, K)), _codes(g, (N, K))
    sa = torch.rand(M, generator=g) * 1e-2 + 1e-4
    sw = torch.rand(N, generator=g) * 1e-2 + 1e-4
    b = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if i % 3 else None
    bb = None if b is None else _gpu.bf16_bits_np(b)
    y = _gpu.scaled_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None if b is None else b.cuda())
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(), bb)
    _gpu.gemm_tolerance_check(y, y_ref, f"fp8 M={M} N={N} K={K}")
    Ai = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
    Wi = torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8)
    yi = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dev = [t.cuda() if t is not None else None for t in (Ai, sa, Wi, sw, b)]  # kept alive through the call
    st = _capi.raw.tfq_scaled_int8_linear(dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(),
                                          dev[3].data_ptr(), None if b is None else dev[4].data_ptr(),
                                          M, N, K, yi.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    yi_ref = oracle.scaled_int8_linear(Ai.numpy(), sa.numpy(), Wi.numpy(), sw.numpy(), bb)
    _gpu.gemm_tolerance_check(yi, yi_ref, f"int8 M={M} N={N} K={K}")


@pytest.mark.parametrize("i", range(len(MX_SHAPES)))
def test_mxfp8_quantizer_and_gemm(i):
    M, N, K = MX_SHAPES[i]
    x = workloads.activations(M, K, seed=3000 + i, nu=4, outlier_cols=2, outlier_mult=40.0, device="cuda")
    w = workloads.weights(N, K, seed=3100 + i, std=0.02, device="cuda")
    b = workloads.bias(N, seed=3200 + i, device="cuda")
    A, sfa = _check_mx_quant(x)
    W, sfw = _check_mx_quant(w)
    y = _gpu.mxfp8_linear(A, sfa, W, sfw, b)
    y_ref = oracle.mxfp8_linear(A.cpu().numpy(), _gpu.mx_untile(sfa.cpu().numpy(), M, K), W.cpu().numpy(),
                                _gpu.mx_untile(sfw.cpu().numpy(), N, K), _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, f"mx M={M} N={N} K={K}")


MULTI_RNG = np.random.default_rng(20261203)
MULTI_CASES = []
while len(MULTI_CASES) < 12:
    n = int(MULTI_RNG.integers(1, 5))
    M = int(MULTI_RNG.integers(1, 3000))
    Ns = [int(MULTI_RNG.integers(0, 160)) * 8 for _ in range(n)]
    K = int(MULTI_RNG.integers(1, 120)) * 16
    if sum(Ns) > 0 and M * sum(Ns) * K <= 2 ** 31:
        MULTI_CASES.append((M, Ns, K, [bool(MULTI_RNG.integers(0, 2)) for _ in range(n)]))
MULTI_CASES.append((1500, [264, 0, 520], 320, [True, False, True]))  # a zero-width Linear between two others


@pytest.mark.parametrize("i", range(len(MULTI_CASES)))
def test_multi_linear_gemms(i):
    """FP8 and INT8 multi-Linear GEMMs on random shapes (N = 0 Linears, null
    biases, rows below and above the CTA-pair threshold): every output equal
    to its single call bit for bit, and within the tolerance of the oracle."""
    import ctypes
    M, Ns, K, with_bias = MULTI_CASES[i]
    g = torch.Generator().manual_seed(4000 + i)
    arr = _capi.pointer_array
    for int8 in (False, True):
        if int8:
            A = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
            Ws = [torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8) for N in Ns]
        else:
            A, Ws = _codes(g, (M, K)), [_codes(g, (N, K)) for N in Ns]
        sa = torch.rand(M, generator=g) * 1e-2 + 1e-4
        sws = [torch.rand(N, generator=g) * 1e-2 + 1e-4 for N in Ns]
        bs = [(torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if wb else None for N, wb in zip(Ns, with_bias)]
        dA, dsa = A.cuda(), sa.cuda()
        dWs, dsws = [w.cuda() for w in Ws], [s.cuda() for s in sws]
        dbs = [None if b is None else b.cuda() for b in bs]
        ys = [_gpu.guarded(M * N, torch.bfloat16, 12345.0) for N in Ns]
        entry = "tfq_scaled_int8_linear_multi" if int8 else "tfq_scaled_fp8_linear_multi"
        st = getattr(_capi.raw, entry)(dA.data_ptr(), dsa.data_ptr(), M, K, len(Ns), arr([w.data_ptr() for w in dWs]),
                                       arr([s.data_ptr() for s in dsws]),
                                       arr([None if b is None else b.data_ptr() for b in dbs]),
                                       (ctypes.c_int64 * len(Ns))(*Ns), arr([y.data_ptr() for y in ys]),
                                       _gpu.stream_handle())
        assert st == _capi.TFQ_OK, _capi.last_error_message()
        _gpu.check_device_error()
        single = _capi.raw.tfq_scaled_int8_linear if int8 else _capi.raw.tfq_scaled_fp8_linear
        ref_fn = oracle.scaled_int8_linear if int8 else oracle.scaled_fp8_linear
        for j, (N, y) in enumerate(zip(Ns, ys)):
            assert torch.all(y[M * N:] == 12345.0), "write past the end of an output"
            if N == 0:
                continue
            y = y[:M * N].view(M, N)
            y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            st = single(dA.data_ptr(), dsa.data_ptr(), dWs[j].data_ptr(), dsws[j].data_ptr(),
                        None if dbs[j] is None else dbs[j].data_ptr(), M, N, K, y1.data_ptr(), _gpu.stream_handle())
            assert st == _capi.TFQ_OK, _capi.last_error_message()
            assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), f"Linear {j} differs from its own call"
            y_ref = ref_fn(A.numpy(), sa.numpy(), Ws[j].numpy(), sws[j].numpy(),
                           None if bs[j] is None else _gpu.bf16_bits_np(bs[j]))
            _gpu.gemm_tolerance_check(y, y_ref, f"{'int8' if int8 else 'fp8'} multi M={M} N={N} K={K} #{j}")
