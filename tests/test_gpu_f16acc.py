"""FP8 GEMM with an FP16 accumulator (NEXT row f3: the fp8-f16-accum mode and
the reduced-qmax study of the LightX2V "模型量化技术" page, section
"MiniMax-H3 FP8 FP16 累加")."""
import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi, workloads
from tests import _gpu

pytestmark = pytest.mark.gpu


def _f16acc(A, sa, W, sw, b):
    M, K = A.shape
    N = W.shape[0]
    out = _gpu.guarded(M * N, torch.bfloat16, 12345.0)
    st = _capi.raw.tfq_scaled_fp8_linear_f16acc(A.data_ptr(), sa.data_ptr(), W.data_ptr(), sw.data_ptr(),
                                                None if b is None else b.data_ptr(), M, N, K, out.data_ptr(),
                                                _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    _gpu.check_device_error()
    assert torch.all(out[M * N:] == 12345.0)
    return out[:M * N].view(M, N)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _gpu.lib()


@pytest.mark.parametrize("M,N,K", [(130, 264, 2048), (777, 520, 1024), (2523, 1992, 256), (9400, 1000, 400)])
def test_integer_sums_are_exact(M, N, K):
    """Codes of +-1 and 0: every partial sum is an integer of magnitude <= K <=
    2048, exact in FP16, so the result matches the oracle to bf16 rounding
    (the third shape runs the pair kernel with its last round split, the
    last two full rounds of pair tiles with ragged M, N and K)."""
    g = torch.Generator().manual_seed(M + N)
    choice = torch.tensor([0x38, 0xB8, 0x00], dtype=torch.uint8)
    A = choice[torch.randint(0, 3, (M, K), generator=g)]
    W = choice[torch.randint(0, 3, (N, K), generator=g)]
    sa = torch.rand(M, generator=g) + 0.5
    sw = torch.rand(N, generator=g) + 0.5
    b = (torch.randn(N, generator=g)).to(torch.bfloat16)
    y = _f16acc(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), b.cuda())
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy(), _gpu.bf16_bits_np(b))
    _gpu.gemm_tolerance_check(y, y_ref, "f16acc integer sums")


def test_error_within_fp16_accumulation_bound():
    """Random small codes (sums stay far below 65504): the error is bounded by
    one FP16 rounding of the running sum per 32-deep MMA step."""
    M, N, K = 300, 264, 1024
    g = torch.Generator().manual_seed(3)
    mag = torch.randint(0x20, 0x48, (M, K), generator=g)            # |a| in [0.125, 3]
    A = (mag | (torch.randint(0, 2, (M, K), generator=g) << 7)).to(torch.uint8)
    magw = torch.randint(0x20, 0x48, (N, K), generator=g)
    W = (magw | (torch.randint(0, 2, (N, K), generator=g) << 7)).to(torch.uint8)
    sa = torch.rand(M, generator=g) * 1e-2 + 1e-3
    sw = torch.rand(N, generator=g) * 1e-2 + 1e-3
    y = _f16acc(A.cuda(), sa.cuda(), W.cuda(), sw.cuda(), None).float().cpu().numpy().astype(np.float64)
    y_ref = oracle.scaled_fp8_linear(A.numpy(), sa.numpy(), W.numpy(), sw.numpy())
    da = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    S = da[A.numpy()] @ da[W.numpy()].T                               # sum_k |a_k w_k|
    bound = (K / 32 + 2) * 2.0 ** -11 * S * np.outer(sa.numpy(), sw.numpy()) + 2.0 ** -8 * np.abs(y_ref) + 1e-9
    assert np.isfinite(y).all()
    assert np.all(np.abs(y - y_ref) <= bound)


# The FP16 accumulator's reading (the pages do not fix the tensor cores'
# accumulation granularity): the running sum is rounded to FP16 once per
# 32-deep MMA step (the K of one kind::f8f6f4 instruction), the step's own
# products summed without FP16 rounding.  FP16_EPS_PER_STEP is twice that
# rounding's relative bound (2^-11), a margin for a step sum rounded to fp32
# first.
FP16_MAX = 65504.0
FP16_EPS_PER_STEP = 2.0 ** -10


def _overflow_verdicts(A, Wq, rows):
    """For sampled rows: which outputs must stay finite and which must
    overflow with an FP16 accumulator, from the oracle's exact running sums
    at every 32-element block of K.  With n steps and eps = n *
    FP16_EPS_PER_STEP, every accumulator value stays within |P_max| (1 + eps) /
    (1 - eps) when no step overflowed (P_max the largest exact running sum
    at a step boundary), so it cannot overflow if that is below FP16_MAX;
    and a final exact sum beyond FP16_MAX (1 + eps) cannot be reached without
    an overflow, after which the sum stays infinite (or NaN)."""
    K = A.shape[1]
    final, pmax = oracle.fp8_block_prefix_sums(A.cpu().numpy(), Wq.cpu().numpy(), 32, rows=rows)
    eps = -(-K // 32) * FP16_EPS_PER_STEP
    must_finite = pmax * (1 + eps) / (1 - eps) < FP16_MAX
    must_overflow = np.abs(final) > FP16_MAX * (1 + eps)
    return must_finite, must_overflow


def test_reduced_qmax_overflow_study(capsys):
    """FFN-out-like Linear (K = 13824 -> N = 5120, X = 4 Student-t(3), FP8
    weights at qmax 448): the fraction of non-finite outputs with an FP16
    accumulator as the activation qmax goes down.  It must fall to zero by
    qmax 7, never rise as qmax decreases, and the FP32-accumulator path must
    stay finite throughout.  On 48 sampled rows (all N) every output the
    oracle's running sums say must stay finite is finite, and every output
    they say must overflow is not (see _overflow_verdicts)."""
    M, K, N = 2048, 13824, 5120
    x = workloads.activations(M, K, seed=41, nu=3, amplitude=4.0, device="cuda")
    w = workloads.weights(N, K, seed=42, std=0.015, device="cuda")
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
    rows = _gpu.sample_rows(M, 47, seed=43)
    ridx = torch.as_tensor(rows, device="cuda")
    fracs, decided = {}, {}
    for qmax in (448.0, 64.0, 21.0, 14.0, 12.0, 7.0):
        A, sa = _gpu.quant_act_fp8(x, qmax)
        y16 = _f16acc(A, sa, Wq, sw, None)
        fracs[qmax] = float((~torch.isfinite(y16.float())).float().mean())
        y32 = _gpu.scaled_linear(A, sa, Wq, sw, None)
        assert torch.isfinite(y32.float()).all()
        must_finite, must_overflow = _overflow_verdicts(A, Wq, rows)
        finite = torch.isfinite(y16[ridx].float()).cpu().numpy()
        assert finite[must_finite].all(), f"qmax {qmax}: an output that cannot overflow is not finite"
        assert not finite[must_overflow].any(), f"qmax {qmax}: an output that must overflow is finite"
        decided[qmax] = (int(must_finite.sum()), int(must_overflow.sum()), int(finite.size))
    with capsys.disabled():
        print("\nFP16-accumulator non-finite fraction by activation qmax:", fracs)
        print("sampled outputs (must stay finite, must overflow, total):", decided)
    qs = sorted(fracs, reverse=True)
    assert all(fracs[a] >= fracs[b] for a, b in zip(qs, qs[1:]))
    assert fracs[7.0] == 0.0 and fracs[448.0] > 0.0
