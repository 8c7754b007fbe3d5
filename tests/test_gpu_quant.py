"""GPU parity of the row quantizers against the oracle: codes and scales
bit-exact, on the workloads' shapes and distributions, ragged sizes and the
degenerate cases (zero rows, K = 0, M = 0, tiny magnitudes, rounding ties)."""
import os

import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi, workloads
from tests import _gpu
from tests._pins import load_hand_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_rows.txt")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _gpu.lib()


def _assert_fp8_equal(x, qmax, rows=None):
    q, s = _gpu.quant_act_fp8(x, qmax)
    q_ref, s_ref = _gpu.oracle_quant_fp8(x, qmax, rows)
    qg = q.cpu().numpy() if rows is None else q[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    sg = s.cpu().numpy() if rows is None else s[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    np.testing.assert_array_equal(sg.view(np.uint32), s_ref.view(np.uint32))
    mism = np.argwhere(qg != q_ref)
    assert mism.size == 0, f"{len(mism)} code mismatches, first {tuple(mism[0])}: gpu {qg[tuple(mism[0])]:#x} " \
                           f"oracle {q_ref[tuple(mism[0])]:#x}"


def test_tiny_config_activation():
    x = workloads.TINY.make_x("x", device="cuda")
    _assert_fp8_equal(x, 448.0)


@pytest.mark.parametrize("qmax", [448.0, 14.0, 7.0, 21.0, 100.0, 12.0])
@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (37, 256), (129, 1024), (65, 3072), (33, 5120),
                                 (17, 12288), (9, 13824), (7, 16384), (130, 20480), (5, 32768), (300, 160), (3, 65536),
                                 (2, 100000)])
def test_ragged_shapes(M, K, qmax):
    """qmax 21 and 100 are not E4M3 numbers (21 is the midpoint of 20 and
    22): the kernel clamps x/s there; for the others it needs no clamp."""
    x = workloads.activations(M, K, seed=M * 7 + K, nu=3, amplitude=4.0, outlier_cols=max(1, K // 100),
                              outlier_mult=30.0, zero_rows=1 if M > 2 else 0, device="cuda")
    _assert_fp8_equal(x, qmax)


def test_quantizer_config_fp8_and_int8():
    """Activation-quantizer workload: [8192, 3072], 1 % outlier columns x50,
    16 all-zero rows; per-token FP8 (448) and per-row INT8 (127)."""
    x = workloads.quantizer_input(device="cuda")
    _assert_fp8_equal(x, 448.0)
    q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)
    zero = (x == 0).all(dim=1)
    assert int(zero.sum()) == 16
    assert torch.all(s[zero] == torch.tensor(np.float32(1e-12) / np.float32(127.0), device="cuda"))


@pytest.mark.parametrize("qmax", [448.0, 14.0, 7.0])
def test_weight_fp8_per_channel(qmax):
    w = workloads.weights(520, 1024, seed=11, std=0.02, device="cuda")
    q, s = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, qmax)
    q_ref, s_ref = _gpu.oracle_quant_fp8(w, qmax)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("K", [16, 256, 5120, 13824, 16384, 24576])
def test_int8_ragged(K):
    x = workloads.activations(77, K, seed=K, nu=4, outlier_cols=3, outlier_mult=20.0, zero_rows=2, device="cuda")
    q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


def test_rounding_edges():
    """Rows built so that x/s hits E4M3 midpoints, subnormals, signed zeros,
    saturation and tiny magnitudes below the 1e-12 floor."""
    grid = torch.tensor(np.r_[0:0x7F].astype(np.uint8)).view(torch.float8_e4m3fn).float()
    mids = (grid[:-1] + grid[1:]) / 2
    row = torch.cat([torch.tensor([448.0]), grid, -grid, mids, -mids, torch.tensor([-0.0, 0.0, 1e-30, -1e-30])])
    K = ((row.numel() + 15) // 16) * 16
    x = torch.zeros(6, K)
    x[0, :row.numel()] = row                       # s = 1: t = x exactly
    x[1, :row.numel()] = row * 2.0 ** -20          # scaled copy (still exact in bf16 where representable)
    x[2, :row.numel()] = row / 448.0 * 14.0
    x[3] = -0.0                                    # all negative zeros
    x[4, :8] = torch.tensor([1e-13, -3e-13, 2e-13, 0, 0, 0, 0, -1e-14])   # below the floor
    x[5, :row.numel()] = row * 3.0                 # a non-power-of-two scale
    x = x.to(torch.bfloat16).cuda()
    for qmax in (448.0, 14.0, 7.0, 21.0, 100.0):
        _assert_fp8_equal(x, qmax)


@pytest.mark.parametrize("K", [16, 5120, 16384])
def test_hand_rows(K):
    """The hand-worked rows of tests/golden/hand_rows.txt (codes derived by
    hand from the formulas and the E4M3FN format), zero-padded to K: the
    padding changes neither the row maximum nor the codes of the given
    values.  K picks the grouped, warp-per-row and staged kernels."""
    for kind, qmax, xs, codes in load_hand_rows(GOLDEN):
        n = len(xs)
        x = torch.zeros(1, K, dtype=torch.float64)
        x[0, :n] = torch.tensor(xs, dtype=torch.float64)
        xb = x.to(torch.bfloat16)
        assert torch.equal(xb[0, :n].double(), x[0, :n]), "hand rows are exact bf16 numbers"
        xd = xb.cuda()
        if kind == "fp8":
            q, s = _gpu.quant_act_fp8(xd, qmax)
            got = [int(c) for c in q[0, :n].cpu()]
        else:
            q, s = _gpu.quant_weight(xd, _capi.TFQ_DTYPE_INT8, qmax)
            got = [int(c) for c in q[0, :n].cpu().view(torch.int8)]
        assert got == codes, (kind, qmax, xs)
        assert torch.all(q[0, n:] == 0)
        amax = max(abs(v) for v in xs)
        assert s.cpu().numpy()[0] == np.float32(max(amax, 1e-12)) / np.float32(qmax)


@pytest.mark.parametrize("K", [16, 5120, 16384])
def test_clamp_of_quotients_above_qmax(K):
    """Rows whose absmax quotient fl32(amax / s) lies one ulp above a qmax that
    is not an E4M3 value (21: between codes 20 and 22; 100: between 96 and
    104), found by search over bf16 magnitudes, in both signs, zero-padded to
    K (grouped, warp-per-row and staged kernels): the clamp brings the
    quotient back to qmax, which ties to the even code; codes and scales are
    compared with the oracle bit for bit."""
    mags = torch.arange(0x3F80, 0x4780, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float().numpy()
    for qmax in (21.0, 100.0):
        s = (mags / np.float32(qmax)).astype(np.float32)
        above = mags[(mags / s).astype(np.float32) > np.float32(qmax)][:24]
        assert len(above) >= 8
        x = torch.zeros(2 * len(above), K, dtype=torch.float32)
        for i, a in enumerate(above):
            x[2 * i, 0], x[2 * i, 1] = float(a), float(a) / 4
            x[2 * i + 1, 0], x[2 * i + 1, 1] = -float(a), float(a) / 8
        xd = x.to(torch.bfloat16).cuda()
        q, sc = _gpu.quant_act_fp8(xd, qmax)
        q_ref, s_ref = _gpu.oracle_quant_fp8(xd, qmax)
        np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
        clamped = int(oracle.e4m3_encode(np.array([qmax], dtype=np.float32))[0])
        assert np.all(q.cpu().numpy()[:, 0] & 0x7F == clamped)


@pytest.mark.parametrize("K", [32, 5120, 16384])
def test_subnormal_inputs(K):
    """bf16 subnormals (below 2^-126): a row of them only (the floored scale),
    among a normal maximum, and next to the smallest normals -- every code 0
    with the input's sign, scales bit-exact, in FP8 and INT8, each kernel."""
    x = torch.zeros(4, K)
    x[0, :4] = torch.tensor([1e-39, -3e-39, 5e-40, -1e-40])
    x[1, :4] = torch.tensor([2.0, -1e-39, 3e-39, -1e-40])
    x[1, -1] = -7e-39
    x[2, :3] = torch.tensor([1e-38, -1.1e-38, 1.17e-38])
    x[3, ::7] = -1e-40
    xd = x.to(torch.bfloat16).cuda()
    assert float(xd.float().abs()[0].max()) < 2.0 ** -126
    for qmax in (448.0, 7.0, 21.0):
        _assert_fp8_equal(xd, qmax)
    q, sc = _gpu.quant_weight(xd, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(xd, 127.0)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


@pytest.mark.parametrize("K", [16, 48, 2048, 3072, 5120, 13824, 16384, 20480, 65536])
def test_absmax_at_row_ends(K):
    """Rows whose absmax is their first or their last element (positive or
    negative), every kernel variant (grouped, warp-per-row of one or several
    segments, staged): the row maximum must cover both ends of the row."""
    x = workloads.activations(16, K, seed=K + 1, nu=4).float()
    peak = x.abs().amax(dim=1) * 3.0
    for r in range(16):
        x[r, -1 if r % 2 == 0 else 0] = peak[r] * (1 if r % 4 < 2 else -1)
    xd = x.to(torch.bfloat16).cuda()
    for qmax in (448.0, 7.0, 21.0):
        _assert_fp8_equal(xd, qmax)
    q, sc = _gpu.quant_weight(xd, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(xd, 127.0)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


@pytest.mark.parametrize("K", [256, 5120, 16384])
@pytest.mark.parametrize("qmax", [1.0, 2.0, 448.0])
def test_huge_magnitude_rows(qmax, K):
    """Rows near the bf16 maximum and rows whose scale is near 2^64: above it
    the kernel takes its IEEE-division branch for the row (grouped,
    one-warp-per-row and shared-memory-staged kernels)."""
    x = workloads.activations(48, K, seed=3, device="cuda").float()
    x[:20] *= 3.0e38 / x[:20].abs().amax(dim=1, keepdim=True)
    x[20:30] *= 1.0e30
    # scales on both sides of 2^64, where the reciprocal-based division hands over to __fdiv_rn
    near = torch.tensor([0.5, 0.99, 0.999, 1.0, 1.001, 1.01, 2.0, 1.0], device="cuda")[:, None]
    x[40:48] *= near * (2.0 ** 64) * qmax / x[40:48].abs().amax(dim=1, keepdim=True)
    x = x.to(torch.bfloat16)
    assert torch.isfinite(x.float()).all()
    _assert_fp8_equal(x, qmax)


def test_empty_and_k0():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    st = _capi.raw.tfq_quant_act_fp8_per_token(x.data_ptr(), 0, 64, 448.0, 0, 0, _gpu.stream_handle())
    assert st == _capi.TFQ_OK
    s = torch.full((5,), -1.0, device="cuda")
    x0 = torch.empty((5, 0), dtype=torch.bfloat16, device="cuda")
    q0 = torch.empty((5, 0), dtype=torch.uint8, device="cuda")
    st = _capi.raw.tfq_quant_act_fp8_per_token(x0.data_ptr() or 16, 5, 0, 7.0, q0.data_ptr() or 16, s.data_ptr(),
                                                _gpu.stream_handle())
    assert st == _capi.TFQ_OK
    _gpu.check_device_error()
    assert torch.all(s == torch.tensor(np.float32(1e-12) / np.float32(7.0), device="cuda"))


@pytest.mark.parametrize("name", ["image_dit_block", "video_dit_block", "reduced_qmax_ffn_out"])
def test_full_size_activations_sampled(name):
    """Full-size DiT activations, bench launch configuration; the oracle
    checks a seeded sample of rows plus the ragged tail."""
    wl = workloads.WORKLOADS[name]
    for xname in sorted(wl.x_shapes()):
        x = wl.make_x(xname, device="cuda")
        rows = _gpu.sample_rows(wl.M, 384, seed=len(xname))
        for qmax in wl.act_qmax:
            _assert_fp8_equal(x, qmax, rows)
        del x
        torch.cuda.empty_cache()


def test_tensor_wrappers_match_raw():
    x = workloads.activations(100, 512, seed=5, device="cuda")
    q1, s1 = _gpu.quant_act_fp8(x, 14.0)
    from int8_w8a8_quantized_b200 import tfq_quant_act_fp8_per_token
    q2, s2 = tfq_quant_act_fp8_per_token(x, 14.0)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1, s2)


@pytest.mark.parametrize("K", [16, 32, 48, 64, 96, 112, 128])
@pytest.mark.parametrize("M", [1, 3, 37, 1000, 4097])
def test_short_rows_sub_warp(M, K):
    """K <= 128 runs the grouped kernel with 2..4 lanes per row and 1 or 4
    units per lane (8..16 rows per warp): ragged M, lane slots beyond the
    row's units, FP8 with and without the clamp, INT8."""
    x = workloads.activations(M, K, seed=M + K, nu=3, outlier_cols=1, outlier_mult=25.0,
                              zero_rows=1 if M > 2 else 0, device="cuda")
    for qmax in (448.0, 21.0):
        _assert_fp8_equal(x, qmax)
    q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


def test_kv_cache_per_vector_full_size():
    """Per-vector FP8 KV cache: one fp32 scale per head_dim vector -- the video
    DiT's K projection viewed as [75600 tokens x 40 heads, 128]; sampled rows."""
    x = workloads.activations(75600 * 40, 128, seed=77, nu=4, device="cuda")
    rows = _gpu.sample_rows(x.shape[0], 4096, seed=78)
    _assert_fp8_equal(x, 448.0, rows)


@pytest.mark.parametrize("K", [144, 256, 272, 384, 512, 528, 1024, 1152, 1536, 2048, 2064])
@pytest.mark.parametrize("M", [1, 5, 130, 2049])
def test_mid_rows_grouped(M, K):
    """128 < K <= 2048 runs the grouped kernel (several rows per warp, up to 8
    units per lane, a row's lanes reduce among themselves); K = 2064 is the
    first size past it.  Ragged M (a warp's last rows missing), units that do
    not fill the row's lanes, FP8 with and without the clamp, INT8."""
    x = workloads.activations(M, K, seed=3 * M + K, nu=3, outlier_cols=2, outlier_mult=25.0,
                              zero_rows=1 if M > 2 else 0, device="cuda")
    for qmax in (448.0, 21.0, 7.0):
        _assert_fp8_equal(x, qmax)
    q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)


@pytest.mark.parametrize("M,K", [(40000, 3072), (33000, 2176)])
def test_many_short_rows_sampled(M, K):
    """More than 32768 rows of K <= 3072 take the two-CTA-per-SM warp-per-row
    variant (fewer rows take the three-CTA one); sampled rows + the tail."""
    x = workloads.activations(M, K, seed=M + K, nu=4, outlier_cols=K // 100, outlier_mult=20.0, zero_rows=3,
                              device="cuda")
    rows = _gpu.sample_rows(M, 512, seed=K)
    _assert_fp8_equal(x, 448.0, rows)
    _assert_fp8_equal(x, 21.0, rows)


@pytest.mark.parametrize("K", [4112, 5120, 5136, 6400, 7680, 10240, 12800])
@pytest.mark.parametrize("M", [3, 300])
def test_segment_choice_boundaries(M, K):
    """Row lengths around the 16- / 20-unit segment choice of the
    warp-per-row kernel: one 20-unit segment (K = 4112, 5120), two
    (10240), three (12800), and lengths where 16 units waste less (5136,
    6400, 7680); FP8 with and without the clamp, INT8."""
    x = workloads.activations(M, K, seed=M * 11 + K, nu=3, outlier_cols=3, outlier_mult=30.0,
                              zero_rows=1 if M > 2 else 0, device="cuda")
    for qmax in (448.0, 21.0):
        _assert_fp8_equal(x, qmax)
    q, s = _gpu.quant_weight(x, _capi.TFQ_DTYPE_INT8, 127.0)
    q_ref, s_ref = _gpu.oracle_quant_int8(x, 127.0)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().view(np.int8), q_ref)
