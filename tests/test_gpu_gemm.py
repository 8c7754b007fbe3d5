"""GPU parity of the scaled FP8 GEMM against the oracle, within the stated
tolerance |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref) element by element:
full comparisons on small and ragged shapes, sampled rows at the full DiT
sizes (same launch configuration as the benchmark)."""
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


def _rand_codes(gen, shape, max_code=0x6F):
    """Finite E4M3 codes with magnitudes up to dec(max_code), random signs."""
    mag = torch.randint(0, max_code + 1, shape, generator=gen, dtype=torch.int32)
    sign = torch.randint(0, 2, shape, generator=gen, dtype=torch.int32) << 7
    return (mag | sign).to(torch.uint8)


def _run_case(M, N, K, with_bias, seed):
    g = torch.Generator().manual_seed(seed)
    A = _rand_codes(g, (M, K))
    W = _rand_codes(g, (N, K))
    sa = (torch.rand(M, generator=g) * 0.01 + 1e-4).float()
    sw = (torch.rand(N, generator=g) * 0.01 + 1e-4).float()
    bias = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if with_bias else None
    y = _gpu.scaled_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None if bias is None else bias.cuda())
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(),
                                     None if bias is None else _gpu.bf16_bits_np(bias))
    return _gpu.gemm_tolerance_check(y, y_ref, f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (1, 8, 16), (100, 136, 48), (129, 264, 144),
                                   (300, 520, 1024), (257, 256, 32), (64, 128, 256), (640, 1024, 2048)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_ragged_full_compare(M, N, K, with_bias):
    _run_case(M, N, K, with_bias, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(512, 256, 128), (513, 264, 144), (777, 520, 1024), (1024, 136, 48),
                                   (2128, 1032, 512), (3000, 3072, 256)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_pair_kernel_full_compare(M, N, K, with_bias):
    """M >= 512 runs the CTA-pair (cta_group::2) kernel: 256-row tiles split
    over two SMs, ragged M (a CTA of the last pair may have no valid rows),
    ragged N inside a 256-column tile, K tails."""
    _run_case(M, N, K, with_bias, seed=7 * M + N + K)


def test_many_tiles_persistent():
    """More tiles than SMs, several tiles per CTA, both accumulator buffers."""
    _run_case(1100, 2048, 512, True, seed=3)


def test_tiny_config_end_to_end():
    """Tiny W8A8 Linear: X [64,256], W [128,256] N(0,0.02), qmax 448, bias."""
    wl = workloads.TINY
    lin = wl.linears[0]
    x = wl.make_x("x", device="cuda")
    w = wl.make_w(lin, device="cuda")
    b = wl.make_bias(lin, device="cuda")
    A, sa = _gpu.quant_act_fp8(x, 448.0)
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
    A_ref, sa_ref = _gpu.oracle_quant_fp8(x, 448.0)
    W_ref, sw_ref = _gpu.oracle_quant_fp8(w, 448.0)
    np.testing.assert_array_equal(A.cpu().numpy(), A_ref)
    np.testing.assert_array_equal(Wq.cpu().numpy(), W_ref)
    np.testing.assert_array_equal(sa.cpu().numpy(), sa_ref)
    np.testing.assert_array_equal(sw.cpu().numpy(), sw_ref)
    y = _gpu.scaled_linear(A, sa, Wq, sw, b)
    y_ref = oracle.scaled_fp8_linear(A_ref, sa_ref, W_ref, sw_ref, _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "tiny")


def test_extreme_codes():
    """Largest codes (+-448) everywhere: sums up to K * 448^2 stay exact-ish in fp32."""
    M, N, K = 130, 264, 512
    A = torch.full((M, K), 0x7E, dtype=torch.uint8)
    A[::2, ::3] = 0xFE
    W = torch.full((N, K), 0x7E, dtype=torch.uint8)
    W[1::2, 1::5] = 0x01  # smallest subnormal
    sa = torch.full((M,), 1e-3)
    sw = torch.full((N,), 2e-3)
    y = _gpu.scaled_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None)
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy())
    _gpu.gemm_tolerance_check(y, y_ref, "extreme")


def test_zero_activation_gives_bias():
    M, N, K = 200, 264, 64
    A = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    W = _rand_codes(torch.Generator().manual_seed(1), (N, K)).cuda()
    b = (torch.randn(N) * 3).to(torch.bfloat16).cuda()
    y = _gpu.scaled_linear(A, torch.ones(M, device="cuda"), W, torch.ones(N, device="cuda"), b)
    assert torch.equal(y, b.expand(M, N))


@pytest.mark.parametrize("name", ["image_dit_block", "video_dit_block", "reduced_qmax_ffn_out"])
def test_full_size_linears_sampled(name):
    """Every Linear of the DiT workloads at full size: GPU quantizer + GPU
    GEMM in the benchmark's launch configuration; the oracle recomputes, over
    all N columns, one row of every 128-row CTA share of every M tile, 512
    more seeded rows and the whole ragged tail."""
    wl = workloads.WORKLOADS[name]
    xs = {}
    for lin in wl.linears:
        if lin.x not in xs:
            xs[lin.x] = wl.make_x(lin.x, device="cuda")
        x = xs[lin.x]
        w = wl.make_w(lin, device="cuda")
        b = wl.make_bias(lin, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        rows = _gpu.tile_sample_rows(wl.M, seed=lin.N + lin.K)
        for qmax in wl.act_qmax:
            A, sa = _gpu.quant_act_fp8(x, qmax)
            y = _gpu.scaled_linear(A, sa, Wq, sw, b)
            ridx = torch.as_tensor(rows, device="cuda")
            y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), Wq.cpu().numpy(),
                                             sw.cpu().numpy(), None if b is None else _gpu.bf16_bits_np(b),
                                             rows=rows)
            _gpu.gemm_tolerance_check(y[ridx], y_ref, f"{name}/{lin.name}/q{qmax:g}")
            del A, sa, y
        del w, Wq
    del xs
    torch.cuda.empty_cache()


def test_tensor_wrapper_linear():
    from int8_w8a8_quantized_b200 import tfq_quant_weight_per_channel, w8a8_linear
    x = workloads.activations(300, 512, seed=9, device="cuda")
    w = workloads.weights(264, 512, seed=10, std=0.02, device="cuda")
    b = workloads.bias(264, seed=11, device="cuda")
    Wq, sw = tfq_quant_weight_per_channel(w, "fp8")
    y = w8a8_linear(x, Wq, sw, b, qmax=448.0)
    A_ref, sa_ref = _gpu.oracle_quant_fp8(x, 448.0)
    y_ref = oracle.scaled_fp8_linear(A_ref, sa_ref, Wq.cpu().numpy(), sw.cpu().numpy(), _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "wrapper")


@pytest.mark.parametrize("entry", ["tfq_scaled_fp8_linear", "tfq_scaled_fp8_linear_f16acc",
                                   "tfq_scaled_fp8_linear_noalloc"])
def test_gemm_tensor_wrappers_match_raw(entry):
    """The tensor-level wrappers pass their operands to the C entry point of
    the same name unchanged: same bits as the raw call (activations at qmax
    7, where the FP16-accumulator GEMM is defined too)."""
    import int8_w8a8_quantized_b200 as pkg
    M, N, K = 300, 264, 512
    x = workloads.activations(M, K, seed=12, device="cuda")
    w = workloads.weights(N, K, seed=13, std=0.02, device="cuda")
    b = workloads.bias(N, seed=14, device="cuda")
    A, sa = _gpu.quant_act_fp8(x, 7.0)
    Wq, sw = pkg.tfq_quant_weight_per_channel(w, "fp8")
    y = getattr(pkg, entry)(A, sa, Wq, sw, b)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = getattr(_capi.raw, entry)(A.data_ptr(), sa.data_ptr(), Wq.data_ptr(), sw.data_ptr(), b.data_ptr(),
                                   M, N, K, out.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    assert torch.equal(y.view(torch.int16), out.view(torch.int16))
    if entry != "tfq_scaled_fp8_linear_f16acc":
        y_ref = oracle.scaled_fp8_linear(A.cpu().numpy(), sa.cpu().numpy(), Wq.cpu().numpy(), sw.cpu().numpy(),
                                         _gpu.bf16_bits_np(b))
        _gpu.gemm_tolerance_check(y, y_ref, entry)


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 256), (3000, 5120, 384)])
def test_pair_kernel_several_tiles_per_cluster(M, N, K):
    """256 / 240 pair tiles over the 74 clusters: every cluster runs 3-4
    tiles, so both TMEM accumulators are reused and the cluster pacing,
    the band raster and the accumulator hand-over run for real; full compare."""
    _run_case(M, N, K, True, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(2523, 1864, 400), (2523, 1992, 256), (4096, 4096, 256), (6889, 3072, 384)])
def test_pair_kernel_split_last_round(M, N, K):
    """Shapes whose last round holds at most half as many tiles as there are
    clusters (80 of 74, 256, 324 tiles): the last round's tiles run as two
    half-width tiles on two clusters each.  Ragged N puts the split on a
    partial tile (72 valid columns: the second half is empty; 200: the second
    half holds 72), ragged M and K tails; full compare."""
    _run_case(M, N, K, True, seed=5 * M + N + K)


def test_float8_views_accepted():
    """The Python binding takes torch.float8_e4m3fn tensors wherever it takes
    E4M3 codes as uint8 (the same bytes): outputs identical to the uint8 path."""
    from int8_w8a8_quantized_b200 import tfq_quant_act_fp8_per_token, tfq_quant_weight_per_channel, \
        tfq_scaled_fp8_linear
    x = workloads.activations(600, 512, seed=21, device="cuda")
    w = workloads.weights(264, 512, seed=22, std=0.02, device="cuda")
    b = workloads.bias(264, seed=23, device="cuda")
    Wq, sw = tfq_quant_weight_per_channel(w, "fp8")
    Wq8 = torch.empty((264, 512), dtype=torch.float8_e4m3fn, device="cuda")
    _, sw8 = tfq_quant_weight_per_channel(w, "fp8", q=Wq8)
    A, sa = tfq_quant_act_fp8_per_token(x)
    A8 = torch.empty((600, 512), dtype=torch.float8_e4m3fn, device="cuda")
    tfq_quant_act_fp8_per_token(x, q=A8)
    assert torch.equal(Wq8.view(torch.uint8), Wq) and torch.equal(sw8, sw)
    assert torch.equal(A8.view(torch.uint8), A)
    y = tfq_scaled_fp8_linear(A, sa, Wq, sw, b)
    y8 = tfq_scaled_fp8_linear(A8, sa, Wq8, sw, b)
    assert torch.equal(y, y8)
    with pytest.raises(TypeError):
        tfq_scaled_fp8_linear(A.view(torch.int8), sa, Wq, sw, b)
    with pytest.raises(ValueError):
        tfq_scaled_fp8_linear(A, sa.cpu(), Wq, sw, b)


@pytest.mark.parametrize("M,N,K", [(100, 136, 65536), (600, 264, 65536), (2048, 1024, 32784)])
def test_long_k_full_compare(M, N, K):
    """Hundreds of K blocks per tile (512 at K = 65536): the stage ring's
    phases wrap many times within one tile; K = 32784 leaves a 16-element
    K tail; one-CTA and pair kernels; full compare."""
    _run_case(M, N, K, True, seed=M + N + K)


# Large pair-kernel shapes, one row of every 128-row CTA share compared: 148
# tiles (two rounds) with 2 K blocks; ragged M, N (the last N tile 232
# columns wide) and K; 444 tiles (six rounds) with a single K block; 592
# tiles (eight rounds) with 8 K blocks.
LARGE_SHAPES = [(9472, 1024, 256), (9400, 1000, 400), (18944, 1536, 128), (9472, 4096, 1024)]


@pytest.mark.parametrize("M,N,K", LARGE_SHAPES)
def test_pair_kernel_large_sampled(M, N, K):
    """One row of every 128-row CTA share, 512 more seeded rows and the
    ragged tail, all N columns, against the oracle."""
    g = torch.Generator().manual_seed(M + N + K)
    A = _rand_codes(g, (M, K))
    W = _rand_codes(g, (N, K))
    sa = (torch.rand(M, generator=g) * 0.01 + 1e-4).float()
    sw = (torch.rand(N, generator=g) * 0.01 + 1e-4).float()
    bias = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16)
    y = _gpu.scaled_linear(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), bias.cuda())
    rows = _gpu.tile_sample_rows(M, seed=M + K)
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(), _gpu.bf16_bits_np(bias),
                                     rows=rows)
    _gpu.gemm_tolerance_check(y[torch.as_tensor(rows, device="cuda")], y_ref, f"M={M} N={N} K={K}")
