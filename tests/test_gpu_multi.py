"""GPU parity of tfq_scaled_fp8_linear_multi and tfq_scaled_int8_linear_multi:
the scaled FP8 (INT8) GEMMs of up to four Linears that share their input, as
one launch of the CTA-pair kernel (their N tiles concatenated) from 512 rows
up.

Each output must equal, bit for bit, the output of the separate
tfq_scaled_fp8_linear (tfq_scaled_int8_linear) call -- the same tiles, the
same arithmetic -- and be within |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref)
of the oracle.
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


def _codes(g, shape):
    mag = torch.randint(0, 0x70, shape, generator=g, dtype=torch.int32)
    return (mag | (torch.randint(0, 2, shape, generator=g, dtype=torch.int32) << 7)).to(torch.uint8).cuda()


def _multi(A, sa, Ws, sws, biases, entry="tfq_scaled_fp8_linear_multi"):
    """The raw C call, guard elements after every output."""
    M, K = A.shape
    n = len(Ws)
    outs = [_gpu.guarded(M * W.shape[0], torch.bfloat16, 12345.0) for W in Ws]
    arr = _capi.pointer_array
    import ctypes
    st = getattr(_capi.raw, entry)(
        A.data_ptr(), sa.data_ptr(), M, K, n, arr([W.data_ptr() for W in Ws]), arr([s.data_ptr() for s in sws]),
        arr([None if b is None else b.data_ptr() for b in biases]), (ctypes.c_int64 * n)(*[W.shape[0] for W in Ws]),
        arr([o.data_ptr() for o in outs]), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    res = []
    for o, W in zip(outs, Ws):
        N = W.shape[0]
        assert torch.all(o[M * N:] == 12345.0), "write past the end of an output"
        res.append(o[:M * N].view(M, N))
    return res


def _case(M, Ns, K, bias_mask, seed, oracle_rows=True):
    g = torch.Generator().manual_seed(seed)
    A = _codes(g, (M, K))
    sa = (torch.rand(M, generator=g) * 0.01 + 1e-4).cuda()
    Ws = [_codes(g, (N, K)) for N in Ns]
    sws = [(torch.rand(N, generator=g) * 0.01 + 1e-4).cuda() for N in Ns]
    biases = [(torch.randn(N, generator=g) * 0.5).to(torch.bfloat16).cuda() if use else None
              for N, use in zip(Ns, bias_mask)]
    ys = _multi(A, sa, Ws, sws, biases)
    rows = _gpu.tile_sample_rows(M, seed=seed) if oracle_rows else None
    for i, (y, W, sw, b) in enumerate(zip(ys, Ws, sws, biases)):
        y1 = _gpu.scaled_linear(A, sa, W, sw, b)
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), f"Linear {i} differs from its own call"
        if oracle_rows:
            y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), W.cpu().numpy(), sw.cpu().numpy(),
                                             None if b is None else _gpu.bf16_bits_np(b), rows=rows)
            _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, f"M={M} Ns={Ns} #{i}")


@pytest.mark.parametrize("M,Ns,K,bias_mask", [
    (6889, [3072, 3072, 3072], 3072, [True, True, True]),      # the image-DiT Q, K, V: 972 tiles
    (2600, [1032, 520, 264], 1024, [True, False, True]),       # ragged N, one Linear without bias
    (2523, [1864, 200, 1992, 8], 400, [True, True, False, True]),  # four Linears, tiny and ragged N, K tail
    (4096, [2048], 512, [True]),                                # one Linear
    (512, [256, 256], 128, [False, False]),                    # smallest pair size, no bias
    (300, [520, 264], 1024, [True, True]),                      # below 512 rows: one launch per Linear
])
def test_multi_matches_single_calls_and_oracle(M, Ns, K, bias_mask):
    _case(M, Ns, K, bias_mask, seed=M + sum(Ns) + K)


def test_zero_width_linear_skipped():
    g = torch.Generator().manual_seed(3)
    M, K = 1024, 256
    A = _codes(g, (M, K))
    sa = (torch.rand(M, generator=g) * 0.01).cuda()
    W0, W1 = _codes(g, (264, K)), _codes(g, (0, K))
    sw0, sw1 = (torch.rand(264, generator=g) * 0.01).cuda(), torch.empty(0, device="cuda")
    y0, y1 = _multi(A, sa, [W0, W1], [sw0, sw1], [None, None])
    assert y1.numel() == 0
    assert torch.equal(y0.view(torch.int16), _gpu.scaled_linear(A, sa, W0, sw0, None).view(torch.int16))


def test_tensor_wrapper():
    from int8_w8a8_quantized_b200 import tfq_scaled_fp8_linear, tfq_scaled_fp8_linear_multi
    x = workloads.activations(900, 640, seed=71, device="cuda")
    A, sa = _gpu.quant_act_fp8(x, 448.0)
    Ws, sws, bs = [], [], []
    for i, N in enumerate((520, 264, 1032)):
        w = workloads.weights(N, 640, seed=72 + i, std=0.02, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        Ws.append(Wq), sws.append(sw), bs.append(workloads.bias(N, seed=80 + i, device="cuda"))
    ys = tfq_scaled_fp8_linear_multi(A, sa, Ws, sws, bs)
    for y, W, sw, b in zip(ys, Ws, sws, bs):
        assert torch.equal(y.view(torch.int16), tfq_scaled_fp8_linear(A, sa, W, sw, b).view(torch.int16))


def test_video_dit_qkv_full_size():
    """The video-DiT block's Q, K and V (75600 x 5120 -> 3 x 5120) as one
    launch: every output bit equal to the three separate calls, and the
    tile-share sample of each within the tolerance of the oracle."""
    wl = workloads.WORKLOADS["video_dit_block"]
    x = wl.make_x("x_attn", device="cuda")
    A, sa = _gpu.quant_act_fp8(x, 448.0)
    del x
    lins = [l for l in wl.linears if l.x == "x_attn"]
    Ws, sws, bs = [], [], []
    for lin in lins:
        w = wl.make_w(lin, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        del w
        Ws.append(Wq), sws.append(sw), bs.append(wl.make_bias(lin, device="cuda"))
    ys = _multi(A, sa, Ws, sws, bs)
    rows = _gpu.tile_sample_rows(wl.M, seed=17)
    ridx = torch.as_tensor(rows, device="cuda")
    for lin, y, W, sw, b in zip(lins, ys, Ws, sws, bs):
        y1 = _gpu.scaled_linear(A, sa, W, sw, b)
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), lin.name
        del y1
        y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), W.cpu().numpy(), sw.cpu().numpy(),
                                         _gpu.bf16_bits_np(b), rows=rows)
        _gpu.gemm_tolerance_check(y[ridx], y_ref, f"video {lin.name}")
    del ys
    torch.cuda.empty_cache()


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


@pytest.mark.parametrize("M,Ns,K,bias_mask", [
    (6889, [3072, 3072, 3072], 3072, [True, True, True]),      # the image-DiT Q, K, V
    (2600, [1032, 520, 264], 1024, [True, False, True]),       # ragged N, one Linear without bias
    (1100, [8, 1864], 400, [False, True]),                     # tiny N, K tail
    (300, [520, 264], 1024, [True, True]),                      # below 512 rows: one launch per Linear
])
def test_int8_multi_matches_single_calls_and_oracle(M, Ns, K, bias_mask):
    seed = 7 * M + sum(Ns) + K
    g = torch.Generator().manual_seed(seed)
    A = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8).cuda()
    sa = (torch.rand(M, generator=g) * 1e-3 + 1e-5).cuda()
    Ws = [torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8).cuda() for N in Ns]
    sws = [(torch.rand(N, generator=g) * 1e-3 + 1e-5).cuda() for N in Ns]
    biases = [(torch.randn(N, generator=g) * 0.5).to(torch.bfloat16).cuda() if use else None
              for N, use in zip(Ns, bias_mask)]
    ys = _multi(A, sa, Ws, sws, biases, entry="tfq_scaled_int8_linear_multi")
    rows = _gpu.tile_sample_rows(M, seed=seed)
    for i, (y, W, sw, b) in enumerate(zip(ys, Ws, sws, biases)):
        y1 = _int8_linear(A, sa, W, sw, b)
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), f"INT8 Linear {i} differs from its own call"
        y_ref = oracle.scaled_int8_linear(A.cpu().numpy(), sa.cpu().numpy(), W.cpu().numpy(), sw.cpu().numpy(),
                                          None if b is None else _gpu.bf16_bits_np(b), rows=rows)
        _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, f"int8 multi M={M} #{i}")


def test_int8_tensor_wrapper():
    from int8_w8a8_quantized_b200 import tfq_scaled_int8_linear, tfq_scaled_int8_linear_multi
    g = torch.Generator().manual_seed(11)
    A = torch.randint(-128, 128, (1536, 512), generator=g, dtype=torch.int8).cuda()
    sa = (torch.rand(1536, generator=g) * 1e-3).cuda()
    Ws = [torch.randint(-128, 128, (N, 512), generator=g, dtype=torch.int8).cuda() for N in (768, 256)]
    sws = [(torch.rand(W.shape[0], generator=g) * 1e-3).cuda() for W in Ws]
    ys = tfq_scaled_int8_linear_multi(A, sa, Ws, sws)
    for y, W, sw in zip(ys, Ws, sws):
        assert torch.equal(y.view(torch.int16), tfq_scaled_int8_linear(A, sa, W, sw).view(torch.int16))


def test_int8_video_dit_qkv_full_size():
    """The INT8 bench's Q/K/V launch at full size: the video-DiT block's
    attention input quantized to INT8 by the GPU quantizer, Q, K and V
    (75600 x 5120 -> 3 x 5120, INT8 weights at 127) as one launch; every
    output bit equal to its single call, and the tile-share sample within the
    tolerance of the oracle's exact integer sums."""
    wl = workloads.WORKLOADS["video_dit_block"]
    x = wl.make_x("x_attn", device="cuda")
    M, K = x.shape
    A = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sa = torch.empty(M, device="cuda")
    st = _capi.raw.tfq_quant_act_int8_per_token(x.data_ptr(), M, K, 127.0, A.data_ptr(), sa.data_ptr(),
                                                 _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    del x
    lins = [l for l in wl.linears if l.x == "x_attn"]
    Ws, sws, bs = [], [], []
    for lin in lins:
        w = wl.make_w(lin, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_INT8, 127.0)
        del w
        Ws.append(Wq.view(torch.int8)), sws.append(sw), bs.append(wl.make_bias(lin, device="cuda"))
    ys = _multi(A, sa, Ws, sws, bs, entry="tfq_scaled_int8_linear_multi")
    rows = _gpu.tile_sample_rows(M, seed=19)
    ridx = torch.as_tensor(rows, device="cuda")
    for lin, y, W, sw, b in zip(lins, ys, Ws, sws, bs):
        y1 = _int8_linear(A, sa, W, sw, b)
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), lin.name
        del y1
        y_ref = oracle.scaled_int8_linear(A.cpu().numpy(), sa.cpu().numpy(), W.cpu().numpy(), sw.cpu().numpy(),
                                          _gpu.bf16_bits_np(b), rows=rows)
        _gpu.gemm_tolerance_check(y[ridx], y_ref, f"int8 video {lin.name}")
    del ys
    torch.cuda.empty_cache()
