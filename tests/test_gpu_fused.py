"""GPU parity of tfq_quant_scaled_fp8_linear, the call that quantizes the
activations per token and runs the scaled FP8 GEMM on them (one kernel from
512 rows up: quantizer warps inside the CTA-pair GEMM).

Its codes and scales must be bit-exact with the oracle's per-token FP8
quantizer, its output within |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref)
of the oracle's GEMM on those codes; and, since it runs the same arithmetic
as the two-call path (row quantizer, then GEMM), every output bit must equal
that path's.
"""
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


def fused(x, Wq, sw, b, qmax, ws=None):
    """The fused call through the raw C ABI, guard bytes after every output."""
    M, K = x.shape
    N = Wq.shape[0]
    A = _gpu.guarded(M * K, torch.uint8, 0xA5)
    sa = _gpu.guarded(M, torch.float32, -7.0)
    y = _gpu.guarded(M * N, torch.bfloat16, 12345.0)
    if ws is None:
        ws = torch.full((_capi.raw.tfq_quant_scaled_fp8_linear_workspace_bytes(M),), 0xEE, dtype=torch.uint8,
                        device="cuda")  # stale contents: the call clears what it uses
    st = _capi.raw.tfq_quant_scaled_fp8_linear(x.data_ptr(), M, K, float(qmax), Wq.data_ptr(), sw.data_ptr(),
                                               None if b is None else b.data_ptr(), N, A.data_ptr(), sa.data_ptr(),
                                               y.data_ptr(), ws.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    assert torch.all(A[M * K:] == 0xA5) and torch.all(sa[M:] == -7.0) and torch.all(y[M * N:] == 12345.0), \
        "write past the end of an output"
    return y[:M * N].view(M, N), A[:M * K].view(M, K), sa[:M]


def two_calls(x, Wq, sw, b, qmax):
    A, sa = _gpu.quant_act_fp8(x, qmax)
    return _gpu.scaled_linear(A, sa, Wq, sw, b), A, sa


def _case(M, N, K, qmax, with_bias, seed, outlier=20.0):
    x = workloads.activations(M, K, seed=seed, outlier_cols=max(1, K // 100), outlier_mult=outlier, device="cuda")
    w = workloads.weights(N, K, seed=seed + 1, std=0.02, device="cuda")
    b = workloads.bias(N, seed=seed + 2, device="cuda") if with_bias else None
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
    return x, Wq, sw, b


def _check_against_oracle(x, Wq, sw, b, qmax, y, A, sa, rows=None, what=""):
    A_ref, sa_ref = _gpu.oracle_quant_fp8(x, qmax, rows)
    A_np = A.cpu().numpy() if rows is None else A[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    s_np = sa.cpu().numpy() if rows is None else sa.cpu().numpy()[rows]
    np.testing.assert_array_equal(A_np, A_ref, err_msg=f"{what}: codes")
    np.testing.assert_array_equal(s_np.view(np.uint32), sa_ref.view(np.uint32), err_msg=f"{what}: scales")
    if rows is None:
        y_ref = oracle.scaled_fp8_linear(A_ref, sa_ref, Wq.cpu().numpy(), sw.cpu().numpy(),
                                         None if b is None else _gpu.bf16_bits_np(b))
        _gpu.gemm_tolerance_check(y, y_ref, what)
    else:
        y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), Wq.cpu().numpy(), sw.cpu().numpy(),
                                         None if b is None else _gpu.bf16_bits_np(b), rows=rows)
        _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, what)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (100, 136, 48), (511, 264, 144),    # below 512: two kernels
                                   (512, 256, 128), (513, 264, 144), (777, 520, 1024), (2128, 1032, 512),
                                   (1100, 2048, 3072), (3000, 520, 5120), (600, 264, 13824)])
@pytest.mark.parametrize("qmax", [448.0, 7.0, 21.0])
def test_ragged_full_compare(M, N, K, qmax):
    """Ragged M (a CTA of the last pair may hold no rows, or a partial share),
    N and K tails, rows of one and of several quantizer segments (K = 13824),
    qmax values that need no clamp (448, 7) and one that does (21)."""
    seed = M + 3 * N + K
    x, Wq, sw, b = _case(M, N, K, qmax, with_bias=(M % 2 == 1), seed=seed)
    y, A, sa = fused(x, Wq, sw, b, qmax)
    _check_against_oracle(x, Wq, sw, b, qmax, y, A, sa, what=f"M={M} N={N} K={K} q={qmax:g}")
    y2, A2, sa2 = two_calls(x, Wq, sw, b, qmax)
    assert torch.equal(A, A2) and torch.equal(sa.view(torch.int32), sa2.view(torch.int32))
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "output differs from the two-call path"


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 256), (6889, 3072, 384), (2523, 1864, 400)])
def test_several_rounds_and_split_last_round(M, N, K):
    """Several tiles per cluster (the quantizer warps must stay ahead of
    every round), and a split last round; full compare."""
    x, Wq, sw, b = _case(M, N, K, 448.0, with_bias=True, seed=M + N)
    y, A, sa = fused(x, Wq, sw, b, 448.0)
    _check_against_oracle(x, Wq, sw, b, 448.0, y, A, sa, what=f"M={M} N={N} K={K}")
    y2, _, _ = two_calls(x, Wq, sw, b, 448.0)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_special_rows():
    """All-zero rows (floored scale), negative zeros, a row whose scale is
    above 2^64 (the IEEE-division branch of the quantizer warps), tiny rows
    below the floor, rows that saturate; bit-exact codes and scales."""
    M, N, K = 1024, 264, 512
    g = torch.Generator().manual_seed(5)
    x = torch.randn(M, K, generator=g)
    x[3] = 0.0
    x[4] = -0.0
    x[5] = torch.randn(K, generator=g) * 1e30
    x[6, :] = 1e-14
    x[7, ::2] = 3.0e38
    x[700:1024:37] = 0.0
    x = x.to(torch.bfloat16).cuda()
    w = workloads.weights(N, K, seed=6, std=0.02, device="cuda")
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
    for qmax in (448.0, 14.0, 100.0):
        y, A, sa = fused(x, Wq, sw, None, qmax)
        A_ref, sa_ref = _gpu.oracle_quant_fp8(x, qmax)
        np.testing.assert_array_equal(A.cpu().numpy(), A_ref)
        np.testing.assert_array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))
        y2, _, _ = two_calls(x, Wq, sw, None, qmax)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_workspace_reused_and_outputs_feed_other_linears():
    """Two calls in a row on one workspace (each clears it first), and the
    codes and scales of a fused call taken by the plain GEMM for the Linears
    that share its input (K and V beside Q)."""
    M, K = 2600, 1024
    x = workloads.activations(M, K, seed=31, outlier_cols=10, outlier_mult=20.0, device="cuda")
    ws = torch.empty((_capi.raw.tfq_quant_scaled_fp8_linear_workspace_bytes(M),), dtype=torch.uint8, device="cuda")
    outs = []
    for i, N in enumerate((1032, 520)):
        w = workloads.weights(N, K, seed=40 + i, std=0.02, device="cuda")
        b = workloads.bias(N, seed=50 + i, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        y, A, sa = fused(x, Wq, sw, b, 448.0, ws=ws)
        y2, A2, sa2 = two_calls(x, Wq, sw, b, 448.0)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
        outs.append((A, sa))
        w3 = workloads.weights(264, K, seed=60 + i, std=0.02, device="cuda")
        W3, sw3 = _gpu.quant_weight(w3, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        y3 = _gpu.scaled_linear(A, sa, W3, sw3, None)
        y3_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), W3.cpu().numpy(), sw3.cpu().numpy())
        _gpu.gemm_tolerance_check(y3, y3_ref, "shared input")
    assert torch.equal(outs[0][0], outs[1][0])


def test_quantize_only_when_n_is_zero():
    x = workloads.activations(700, 256, seed=3, device="cuda")
    M, K = x.shape
    A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    ws = torch.empty((_capi.raw.tfq_quant_scaled_fp8_linear_workspace_bytes(M),), dtype=torch.uint8, device="cuda")
    st = _capi.raw.tfq_quant_scaled_fp8_linear(x.data_ptr(), M, K, 448.0, None, None, None, 0, A.data_ptr(),
                                               sa.data_ptr(), None, ws.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    A_ref, sa_ref = _gpu.oracle_quant_fp8(x, 448.0)
    np.testing.assert_array_equal(A.cpu().numpy(), A_ref)
    np.testing.assert_array_equal(sa.cpu().numpy(), sa_ref)


def test_tensor_wrapper_matches_raw_call():
    from int8_w8a8_quantized_b200 import tfq_quant_scaled_fp8_linear
    x, Wq, sw, b = _case(900, 520, 640, 448.0, with_bias=True, seed=77)
    y, A, sa = tfq_quant_scaled_fp8_linear(x, Wq, sw, b, qmax=448.0)
    y2, A2, sa2 = fused(x, Wq, sw, b, 448.0)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16)) and torch.equal(A, A2) and torch.equal(sa, sa2)


@pytest.mark.parametrize("name", ["image_dit_block", "video_dit_block", "reduced_qmax_ffn_out"])
def test_full_size_linears(name):
    """Every Linear of the DiT workloads at full size through the fused call,
    in the benchmark's launch configuration: codes, scales and every output
    bit equal to the two-call path's over the whole tensors; codes and scales
    of sampled rows bit-exact with the oracle, and their outputs (all N) within
    the tolerance of the oracle's GEMM -- one row of every 128-row CTA share,
    512 more seeded rows and the ragged tail."""
    wl = workloads.WORKLOADS[name]
    xs = {}
    for lin in wl.linears:
        if lin.x not in xs:
            xs[lin.x] = wl.make_x(lin.x, device="cuda")
        x = xs[lin.x]
        w = wl.make_w(lin, device="cuda")
        b = wl.make_bias(lin, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        del w
        rows = _gpu.tile_sample_rows(wl.M, seed=lin.N + 2 * lin.K)
        for qmax in wl.act_qmax:
            y, A, sa = fused(x, Wq, sw, b, qmax)
            y2, A2, sa2 = two_calls(x, Wq, sw, b, qmax)
            assert torch.equal(A, A2) and torch.equal(sa.view(torch.int32), sa2.view(torch.int32))
            assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"{name}/{lin.name}: differs"
            del y2, A2, sa2
            _check_against_oracle(x, Wq, sw, b, qmax, y, A, sa, rows=rows, what=f"{name}/{lin.name}/q{qmax:g}")
            del y, A, sa
        del Wq
    del xs
    torch.cuda.empty_cache()
