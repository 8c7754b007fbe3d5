"""Pins for the oracle's per-row quantizers (CPU only).

* hand-worked rows (tests/golden/hand_rows.txt, derived by hand);
* invariants the formulas fix: the absmax element maps to +-qmax, every code
  is within half an E4M3 step (or half an integer) of x/s, INT8 codes stay in
  range, scales are positive and finite, an all-zero row has the floored
  scale and zero codes;
* an independent recomputation: numpy's IEEE fp32 division followed by the
  brute-force grid search of tests/_pins.py (FP8) or numpy's half-to-even
  rint (INT8).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from int8_w8a8_quantized_b200 import workloads
from tests._pins import bf16_bits, bits_to_f32, bruteforce_e4m3, e4m3_spacing, load_hand_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_rows.txt")


def _row_bits(values):
    t = torch.tensor(values, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float64), torch.tensor(values, dtype=torch.float64)), \
        "hand rows must be exact bf16 numbers"
    return bf16_bits(t)[None, :]


@pytest.mark.parametrize("case", load_hand_rows(GOLDEN), ids=lambda c: f"{c[0]}-q{c[1]:g}-{c[2][:2]}")
def test_hand_rows(case):
    kind, qmax, x, codes = case
    bits = _row_bits(x)
    if kind == "fp8":
        q, s = oracle.quant_rows_fp8(bits, qmax)
        assert [int(c) for c in q[0]] == codes
    else:
        q, s = oracle.quant_rows_int8(bits, qmax)
        assert [int(c) for c in q[0]] == codes
    amax = max(abs(v) for v in x)
    assert s[0] == np.float32(max(amax, np.float32(1e-12))) / np.float32(qmax)


def _inputs():
    out = []
    for seed, (M, K) in enumerate([(37, 256), (16, 48), (5, 1024)]):
        x = workloads.activations(M, K, seed=100 + seed, outlier_cols=3, outlier_mult=30.0, zero_rows=2)
        out.append(x)
    out.append(workloads.activations(33, 160, seed=7, nu=3, amplitude=4.0))
    # rows whose absmax is their last element (every other row) or their first: the row maximum must
    # cover the whole row, ends included
    ends = workloads.activations(8, 96, seed=9).to(torch.float32)
    peak = ends.abs().amax(dim=1) * 3.0
    for r in range(8):
        ends[r, -1 if r % 2 == 0 else 0] = peak[r] * (1 if r % 4 < 2 else -1)
    out.append(ends.to(torch.bfloat16))
    # tiny magnitudes (scale near the 1e-12 floor) and a row of negative zeros
    tiny = workloads.activations(4, 64, seed=8) * 1e-13
    tiny[3] = -0.0
    out.append(tiny.to(torch.bfloat16))
    return out


@pytest.mark.parametrize("qmax", [448.0, 14.0, 7.0, 21.0, 100.0])
def test_fp8_invariants_and_recompute(qmax):
    for x in _inputs():
        bits = bf16_bits(x)
        xf = bits_to_f32(bits)
        q, s = oracle.quant_rows_fp8(bits, qmax)
        amax = np.abs(xf).max(axis=1)
        s_ref = np.maximum(amax, np.float32(1e-12)).astype(np.float32) / np.float32(qmax)
        np.testing.assert_array_equal(s, s_ref)
        assert np.all(s > 0) and np.all(np.isfinite(s))
        t = xf / s[:, None]                                   # fp32 IEEE division
        t = np.clip(t, -np.float32(qmax), np.float32(qmax))
        np.testing.assert_array_equal(q, bruteforce_e4m3(t))
        # absmax element -> code of +-qmax (rows whose amax is above the floor)
        qcode = int(bruteforce_e4m3(np.array([qmax]))[0])
        for r in range(x.shape[0]):
            if amax[r] >= 1e-12:
                k = int(np.argmax(np.abs(xf[r])))
                assert int(q[r, k]) & 0x7F == qcode
                assert (int(q[r, k]) >> 7) == (1 if xf[r, k] < 0 else 0)
            else:  # floored scale: the row maps strictly inside +-qmax
                assert np.all((q[r] & 0x7F) <= qcode)
        # dequantization error: |dec(q) - x/s| <= half an E4M3 step at |x/s|
        dec = oracle.e4m3_decode(q)
        tt = xf.astype(np.float64) / s[:, None].astype(np.float64)
        bound = e4m3_spacing(np.minimum(np.abs(tt), qmax)) / 2 * (1 + 2.0 ** -20)
        assert np.all(np.abs(dec - np.clip(tt, -qmax, qmax)) <= bound + 2.0 ** -10)


@pytest.mark.parametrize("qmax,amax", [(21.0, 1.4140625), (100.0, 1.0234375)])
def test_fp8_clamp_of_a_quotient_above_qmax(qmax, amax):
    """A row whose absmax quotient fl32(amax / s) lands one ulp above qmax (a
    qmax that is not an E4M3 value lies halfway between two codes): the clamp
    brings it back to qmax, which ties to the even code, while the unclamped
    quotient would round up to the next code."""
    row = np.array([amax, -amax / 2, amax / 4], dtype=np.float32)
    bits = _row_bits([float(v) for v in row])
    s = np.float32(amax) / np.float32(qmax)
    t = np.float32(amax) / s
    assert t > np.float32(qmax)                       # the case this pins
    clamped, unclamped = bruteforce_e4m3(np.array([qmax], dtype=np.float32))[0], bruteforce_e4m3(np.array([t]))[0]
    assert clamped != unclamped
    q, s_o = oracle.quant_rows_fp8(bits, qmax)
    assert s_o[0] == s and int(q[0, 0]) == int(clamped)
    q_neg, _ = oracle.quant_rows_fp8(_row_bits([float(-v) for v in row]), qmax)
    assert int(q_neg[0, 0]) == int(clamped) | 0x80


def test_fp8_zero_rows_and_negative_zero():
    x = torch.zeros(3, 32, dtype=torch.bfloat16)
    x[1] = -0.0
    x[2, 5] = -1e-30
    q, s = oracle.quant_rows_fp8(bf16_bits(x), 448.0)
    np.testing.assert_array_equal(s, np.full(3, np.float32(1e-12) / np.float32(448.0)))
    assert np.all(q[0] == 0x00) and np.all(q[1] == 0x80)
    # -1e-30 with the floored scale: t = -1e-30 / 2.2e-15 ~ -4.5e-16 -> -0
    assert q[2, 5] == 0x80 and np.all(np.delete(q[2], 5) == 0)


def test_int8_invariants_and_recompute():
    for x in _inputs():
        bits = bf16_bits(x)
        xf = bits_to_f32(bits)
        q, s = oracle.quant_rows_int8(bits, 127.0)
        amax = np.abs(xf).max(axis=1)
        s_ref = np.maximum(amax, np.float32(1e-12)).astype(np.float32) / np.float32(127.0)
        np.testing.assert_array_equal(s, s_ref)
        t = xf / s[:, None]
        np.testing.assert_array_equal(q, np.clip(np.rint(t), -128, 127).astype(np.int8))
        assert q.min() >= -127 and q.max() <= 127
        for r in range(x.shape[0]):
            if amax[r] >= 1e-12:
                k = int(np.argmax(np.abs(xf[r])))
                assert abs(int(q[r, k])) == 127
        err = np.abs(q.astype(np.float64) - xf.astype(np.float64) / s[:, None])
        assert np.all(err <= 0.5 + 1e-5)


def test_rows_are_independent():
    x = workloads.activations(12, 96, seed=3, outlier_cols=2, outlier_mult=20.0)
    bits = bf16_bits(x)
    q, s = oracle.quant_rows_fp8(bits, 448.0)
    for r in (0, 5, 11):
        q1, s1 = oracle.quant_rows_fp8(bits[r:r + 1], 448.0)
        np.testing.assert_array_equal(q1[0], q[r])
        assert s1[0] == s[r]
