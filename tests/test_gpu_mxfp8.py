"""GPU parity of MXFP8 (32-value blocks, E8M0 scales) against the oracle:
quantizer codes and scale codes bit-exact (scale buffer read back through the
documented layout, padding entries checked), block-scaled GEMM within the
GEMM tolerance, on ragged shapes, hand-made scale patterns and the full-size
video-DiT Linears (sampled rows)."""
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


def _check_quant(x):
    R, K = x.shape
    q, sf = _gpu.quant_mxfp8(x)
    q_ref, sf_ref = oracle.quant_mxfp8(_gpu.bf16_bits_np(x))
    sf_host = sf.cpu().numpy()
    got_sf = _gpu.mx_untile(sf_host, R, K)
    mism = np.argwhere(got_sf != sf_ref)
    assert mism.size == 0, f"{len(mism)} scale mismatches, first {tuple(mism[0])}: gpu {got_sf[tuple(mism[0])]} " \
                           f"oracle {sf_ref[tuple(mism[0])]}"
    qg = q.cpu().numpy()
    mism = np.argwhere(qg != q_ref)
    assert mism.size == 0, f"{len(mism)} code mismatches, first {tuple(mism[0])}: gpu {qg[tuple(mism[0])]:#x} " \
                           f"oracle {q_ref[tuple(mism[0])]:#x}"
    pad = np.ones(sf_host.size, dtype=bool)
    pad[_gpu.mx_sf_offsets(R, K).reshape(-1)] = False
    assert np.all(sf_host[pad] == 127), "padding entries must hold code 127"
    return q, sf


@pytest.mark.parametrize("R,K", [(7, 32), (130, 256), (9, 5120)])
def test_block_absmax_at_block_ends(R, K):
    """Blocks whose absmax is their first or their last element (either sign):
    the block maximum, and with it the E8M0 scale, must cover the block's ends."""
    x = workloads.activations(R, K, seed=R + K, nu=4).float()
    xb = x.view(R, K // 32, 32)
    peak = xb.abs().amax(dim=2) * 3.0
    for b in range(K // 32):
        pos = -1 if b % 2 == 0 else 0
        xb[:, b, pos] = peak[:, b] * (1 if b % 4 < 2 else -1)
    _check_quant(x.to(torch.bfloat16).cuda())


@pytest.mark.parametrize("R,K", [(1, 32), (3, 96), (5, 160), (130, 256), (129, 5120), (300, 1056),
                                 (17, 13824), (2049, 128), (64, 4096)])
def test_quant_ragged(R, K):
    x = workloads.activations(R, K, seed=R * 3 + K, nu=3, amplitude=2.0, outlier_cols=max(1, K // 64),
                              outlier_mult=40.0, zero_rows=1 if R > 2 else 0, device="cuda")
    _check_quant(x)


def test_quant_special_blocks():
    """Blocks of zeros and -0, a lone subnormal (scale clamped to code 0),
    magnitudes near the bf16 maximum, saturation (block max in (448, 512)
    after scaling), negative values below the smallest subnormal (-0 code),
    rounding ties; and whole rows spanning 2^-130 .. 2^120."""
    K = 32 * 12
    x = torch.zeros(6, K, dtype=torch.float64)
    x[0, 32:64] = -0.0
    x[0, 64 + 7] = 2.0 ** -130
    x[0, 96:128] = torch.linspace(-3, 3, 32) * 2.0 ** 120
    x[0, 128] = 500.0
    x[0, 129] = 3.0
    x[0, 160] = 256.0
    x[0, 161] = 1.0625
    x[0, 162] = 1.1875
    x[0, 163] = 3 * 2.0 ** -10
    x[0, 164] = -(2.0 ** -10)
    x[0, 165] = -(2.0 ** -14)
    x[1] = torch.exp2(torch.linspace(-130, 120, K)) * torch.where(torch.arange(K) % 3 == 0, -1.0, 1.0)
    g = torch.Generator().manual_seed(3)
    x[2:] = torch.randn(4, K, generator=g, dtype=torch.float64) * torch.exp2(
        torch.randint(-60, 60, (4, K // 32), generator=g).double()).repeat_interleave(32, dim=1)
    xb = x.to(torch.bfloat16).cuda()
    assert torch.isfinite(xb.float()).all()
    _check_quant(xb)


def _rand_codes(gen, shape, max_code=0x7E):
    mag = torch.randint(0, max_code + 1, shape, generator=gen, dtype=torch.int32)
    sign = torch.randint(0, 2, shape, generator=gen, dtype=torch.int32) << 7
    return (mag | sign).to(torch.uint8)


def _gemm_case(M, N, K, with_bias, seed, lo=110, hi=140):
    """Random codes and random scale codes in [lo, hi), placed with the
    layout helper: checks the tensor-core reading of both scale layouts
    independently of the quantizer."""
    g = torch.Generator().manual_seed(seed)
    A = _rand_codes(g, (M, K))
    W = _rand_codes(g, (N, K))
    sa = torch.randint(lo, hi, (M, K // 32), generator=g).to(torch.uint8).numpy()
    sw = torch.randint(lo, hi, (N, K // 32), generator=g).to(torch.uint8).numpy()
    bias = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if with_bias else None
    y = _gpu.mxfp8_linear(A.cuda(), torch.from_numpy(_gpu.mx_tile(sa, K)).cuda(), W.cuda(),
                          torch.from_numpy(_gpu.mx_tile(sw, K)).cuda(), None if bias is None else bias.cuda())
    y_ref = oracle.mxfp8_linear(A.numpy(), sa, W.numpy(), sw, None if bias is None else _gpu.bf16_bits_np(bias))
    _gpu.gemm_tolerance_check(y, y_ref, f"mx M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(128, 192, 128), (1, 8, 32), (100, 136, 96), (129, 200, 160),
                                   (300, 520, 1024), (257, 384, 32), (640, 1032, 2048), (1100, 2048, 512)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_gemm_random_scale_codes(M, N, K, with_bias):
    """Ragged M and N (N tiles of 192 start 0 or 64 rows into a scale atom),
    K tails (K % 128 != 0: padded scale blocks), several tiles per CTA."""
    _gemm_case(M, N, K, with_bias, seed=M + 3 * N + K)


def test_gemm_per_block_scales_matter():
    """One scale code per K block differs wildly between blocks (2^-20 ..
    2^20): a kernel that applied the wrong block's scale, or one scale per
    row, fails by orders of magnitude."""
    _gemm_case(256, 384, 512, True, seed=11, lo=107, hi=148)


def test_quant_then_gemm_tiny_linear():
    wl = workloads.TINY
    lin = wl.linears[0]
    x = wl.make_x("x", device="cuda")
    w = wl.make_w(lin, device="cuda")
    b = wl.make_bias(lin, device="cuda")
    A, sfa = _check_quant(x)
    W, sfw = _check_quant(w)
    y = _gpu.mxfp8_linear(A, sfa, W, sfw, b)
    M, K = x.shape
    N = w.shape[0]
    y_ref = oracle.mxfp8_linear(A.cpu().numpy(), _gpu.mx_untile(sfa.cpu().numpy(), M, K), W.cpu().numpy(),
                                _gpu.mx_untile(sfw.cpu().numpy(), N, K), _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "mx tiny")


def test_full_size_video_linears_sampled():
    """The video-DiT block's Linears in MXFP8 at full size: GPU quantizer
    (sampled rows checked bit-exact) and GPU GEMM (sampled rows within the
    tolerance): one row of every 128-row CTA share of every M tile, 512 more
    seeded rows and the ragged tail, all N columns."""
    wl = workloads.WORKLOADS["video_dit_block"]
    xs = {}
    for lin in wl.linears:
        if lin.x not in xs:
            xs[lin.x] = wl.make_x(lin.x, device="cuda")
        x = xs[lin.x]
        w = wl.make_w(lin, device="cuda")
        b = wl.make_bias(lin, device="cuda")
        M, K = x.shape
        N = w.shape[0]
        A, sfa = _capi.tfq_quant_mxfp8(x)
        W, sfw = _capi.tfq_quant_mxfp8(w)
        y = _capi.tfq_mxfp8_linear(A, sfa, W, sfw, b)
        torch.cuda.synchronize()
        _gpu.check_device_error()
        rows = _gpu.tile_sample_rows(M, seed=lin.N + lin.K)
        ridx = torch.as_tensor(rows, device="cuda")
        xr = x[ridx]
        q_ref, sf_ref = oracle.quant_mxfp8(_gpu.bf16_bits_np(xr))
        np.testing.assert_array_equal(A[ridx].cpu().numpy(), q_ref)
        sfa_rm = _gpu.mx_untile(sfa.cpu().numpy(), M, K)
        np.testing.assert_array_equal(sfa_rm[rows], sf_ref)
        sfw_rm = _gpu.mx_untile(sfw.cpu().numpy(), N, K)
        y_ref = oracle.mxfp8_linear(q_ref, sf_ref, W.cpu().numpy(), sfw_rm, _gpu.bf16_bits_np(b))
        _gpu.gemm_tolerance_check(y[ridx], y_ref, f"mx video/{lin.name}")
        del A, sfa, W, sfw, y, w
    del xs
    torch.cuda.empty_cache()


def test_wrapper_linear():
    from int8_w8a8_quantized_b200 import mxfp8_linear, tfq_quant_mxfp8
    x = workloads.activations(300, 512, seed=9, device="cuda")
    w = workloads.weights(264, 512, seed=10, std=0.02, device="cuda")
    b = workloads.bias(264, seed=11, device="cuda")
    Wq, sfw = tfq_quant_mxfp8(w)
    y = mxfp8_linear(x, Wq, sfw, b)
    A_ref, sfa_ref = oracle.quant_mxfp8(_gpu.bf16_bits_np(x))
    y_ref = oracle.mxfp8_linear(A_ref, sfa_ref, Wq.cpu().numpy(), _gpu.mx_untile(sfw.cpu().numpy(), 264, 512),
                                _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "mx wrapper")


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 128), (2600, 5120, 256)])
def test_gemm_pair_several_tiles_per_cluster(M, N, K):
    """Several 256x256 pair tiles per cluster: both overlapping TMEM
    accumulators are reused, so every tile's first MMA waits for the other
    buffer's shared columns to be read; full compare."""
    _gemm_case(M, N, K, True, seed=M + 7 * N + K)


@pytest.mark.parametrize("M,N,K", [(130, 200, 32768), (700, 520, 16416)])
def test_gemm_long_k(M, N, K):
    """Hundreds of K blocks per tile (and 1024 scale blocks per row): the scale
    atoms of late K steps, the stage ring wrapping many times; K = 16416 ends
    in a partial scale atom; one-CTA and pair kernels."""
    _gemm_case(M, N, K, True, seed=M + N + K)
