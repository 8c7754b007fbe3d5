"""Pins for the oracle's scaled GEMMs (CPU only).

* brute force with exact rational arithmetic (fractions.Fraction) on small
  non-square cases, so a transposed operand or a swapped scale index fails;
* special cases with closed forms: an identity weight, a K = 1 outer
  product, an all-zero activation (the output is the bias), row sampling.
The E4M3 values used by the brute force come from the grid in tests/_pins.py,
not from the oracle's decoder.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._pins import GRID


def _e4m3_value(code: int) -> Fraction:
    mag = Fraction(GRID[code & 0x7F])
    return -mag if code & 0x80 else mag


def _bf16_value(bits: int) -> Fraction:
    return Fraction(float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]))


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38  # no NaN codes
    return c


def _rand_bias_bits(rng, n):
    f = (rng.standard_normal(n) * 0.5).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)  # truncation is fine: any bf16 will do


@pytest.mark.parametrize("M,N,K", [(8, 8, 16), (8, 6, 16), (3, 5, 7), (5, 2, 33)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_bruteforce_rational(M, N, K, with_bias):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    A = _rand_codes(rng, (M, K))
    W = _rand_codes(rng, (N, K))
    sa = rng.uniform(0.001, 2.0, M).astype(np.float32)
    sw = rng.uniform(0.001, 2.0, N).astype(np.float32)
    b = _rand_bias_bits(rng, N) if with_bias else None
    y = oracle.scaled_fp8_linear(A, sa, W, sw, b)
    assert y.shape == (M, N)
    for m in range(M):
        for n in range(N):
            acc = sum(_e4m3_value(int(A[m, k])) * _e4m3_value(int(W[n, k])) for k in range(K))
            prod = acc * Fraction(float(sa[m])) * Fraction(float(sw[n]))
            exact = prod + (_bf16_value(int(b[n])) if b is not None else 0)
            mag = abs(float(prod)) + (abs(float(_bf16_value(int(b[n])))) if b is not None else 0.0)
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(4 * 2.0 ** -53 * mag)


def test_identity_weight():
    rng = np.random.default_rng(5)
    K = 16
    A = _rand_codes(rng, (4, K))
    W = np.zeros((K, K), dtype=np.uint8)
    np.fill_diagonal(W, 0x38)  # 1.0
    sa = np.ones(4, np.float32)
    sw = np.ones(K, np.float32)
    y = oracle.scaled_fp8_linear(A, sa, W, sw)
    expect = np.array([[float(_e4m3_value(int(c))) for c in row] for row in A])
    np.testing.assert_array_equal(y, expect)


def test_k1_outer_product():
    rng = np.random.default_rng(6)
    A = _rand_codes(rng, (6, 1))
    W = _rand_codes(rng, (9, 1))
    sa = rng.uniform(0.1, 1, 6).astype(np.float32)
    sw = rng.uniform(0.1, 1, 9).astype(np.float32)
    y = oracle.scaled_fp8_linear(A, sa, W, sw)
    a = np.array([float(_e4m3_value(int(c))) for c in A[:, 0]]) * sa.astype(np.float64)
    w = np.array([float(_e4m3_value(int(c))) for c in W[:, 0]]) * sw.astype(np.float64)
    np.testing.assert_allclose(y, np.outer(a, w), rtol=4e-16, atol=0)


def test_zero_activation_gives_bias():
    rng = np.random.default_rng(7)
    A = np.zeros((3, 32), np.uint8)
    W = _rand_codes(rng, (10, 32))
    b = _rand_bias_bits(rng, 10)
    y = oracle.scaled_fp8_linear(A, np.ones(3, np.float32), W, np.ones(10, np.float32), b)
    bias = np.array([float(_bf16_value(int(v))) for v in b])
    np.testing.assert_array_equal(y, np.broadcast_to(bias, (3, 10)))


def test_row_sampling_matches_full():
    rng = np.random.default_rng(8)
    A = _rand_codes(rng, (20, 64))
    W = _rand_codes(rng, (12, 64))
    sa = rng.uniform(0.01, 1, 20).astype(np.float32)
    sw = rng.uniform(0.01, 1, 12).astype(np.float32)
    b = _rand_bias_bits(rng, 12)
    full = oracle.scaled_fp8_linear(A, sa, W, sw, b)
    rows = np.array([19, 0, 7, 7])
    part = oracle.scaled_fp8_linear(A, sa, W, sw, b, rows=rows)
    np.testing.assert_array_equal(part, full[rows])


@pytest.mark.parametrize("M,N,K", [(8, 6, 16), (4, 9, 31)])
def test_int8_bruteforce(M, N, K):
    rng = np.random.default_rng(M + N + K)
    A = rng.integers(-128, 128, (M, K), dtype=np.int8)
    W = rng.integers(-128, 128, (N, K), dtype=np.int8)
    sa = rng.uniform(0.001, 2.0, M).astype(np.float32)
    sw = rng.uniform(0.001, 2.0, N).astype(np.float32)
    b = _rand_bias_bits(rng, N)
    y = oracle.scaled_int8_linear(A, sa, W, sw, b)
    for m in range(M):
        for n in range(N):
            acc = sum(int(A[m, k]) * int(W[n, k]) for k in range(K))
            exact = Fraction(acc) * Fraction(float(sa[m])) * Fraction(float(sw[n])) + _bf16_value(int(b[n]))
            mag = abs(acc * float(sa[m]) * float(sw[n])) + abs(float(_bf16_value(int(b[n]))))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(4 * 2.0 ** -53 * mag)


@pytest.mark.parametrize("M,N,K,block", [(3, 4, 70, 32), (2, 5, 64, 32), (4, 3, 33, 16), (2, 2, 31, 32), (3, 3, 9, 1)])
def test_block_prefix_sums_bruteforce(M, N, K, block):
    """The FP16-accumulator study's oracle: the exact running sum at every
    block boundary (a partial last block included), by exact rational
    arithmetic over the independent E4M3 grid; the final sum and the largest
    |running sum| at a boundary.  The codes are mostly large and of one
    sign per row, so intermediate maxima exceed the final sum."""
    rng = np.random.default_rng(M + 10 * N + 100 * K + block)
    A = _rand_codes(rng, (M, K))
    W = _rand_codes(rng, (N, K))
    A[0, : K // 2] = 0x70          # a long positive run, then mixed: the peak lies inside
    W[:, : K // 2] = 0x68
    final, pmax = oracle.fp8_block_prefix_sums(A, W, block)
    assert final.shape == (M, N) and pmax.shape == (M, N)
    for m in range(M):
        for n in range(N):
            acc, peak = Fraction(0), Fraction(0)
            for k in range(K):
                acc += _e4m3_value(int(A[m, k])) * _e4m3_value(int(W[n, k]))
                if (k + 1) % block == 0 or k + 1 == K:
                    peak = max(peak, abs(acc))
            assert Fraction(final[m, n]) == acc
            assert Fraction(pmax[m, n]) == peak
    rows = np.array([M - 1, 0])
    f2, p2 = oracle.fp8_block_prefix_sums(A, W, block, rows=rows)
    np.testing.assert_array_equal(f2, final[rows])
    np.testing.assert_array_equal(p2, pmax[rows])


def test_block_prefix_max_is_not_the_final_sum():
    """A sum that climbs to 16 * 448^2 and comes back to zero: the running
    maximum at block boundaries (block 16) is the peak, the final sum 0."""
    K = 32
    A = np.full((1, K), 0x7E, dtype=np.uint8)           # 448
    W = np.full((1, K), 0x7E, dtype=np.uint8)
    W[0, 16:] = 0xFE                                     # -448
    final, pmax = oracle.fp8_block_prefix_sums(A, W, 16)
    assert final[0, 0] == 0.0 and pmax[0, 0] == 16 * 448.0 ** 2
    final, pmax = oracle.fp8_block_prefix_sums(A, W, 32)
    assert final[0, 0] == 0.0 and pmax[0, 0] == 0.0
