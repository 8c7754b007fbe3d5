"""Pins for the oracle's E4M3FN encoder/decoder (CPU only).

The encoder is checked three independent ways: a brute-force nearest search
over the grid built from the format definition (tests/_pins.py), torch's own
CPU float8_e4m3fn cast (a library routine, in its non-saturating range), and
the exact midpoints between neighbouring codes.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._pins import GRID, bruteforce_e4m3


def test_decode_matches_grid():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes)
    assert np.isnan(dec[0x7F]) and np.isnan(dec[0xFF])
    np.testing.assert_array_equal(dec[:0x7F], GRID)
    np.testing.assert_array_equal(dec[0x80:0xFF], -GRID)
    assert np.signbit(dec[0x80])
    # Every finite code is an exact fp32 number: decode and re-encode.
    finite = np.r_[0:0x7F, 0x80:0xFF].astype(np.uint8)
    back = oracle.e4m3_encode(dec[finite].astype(np.float32))
    np.testing.assert_array_equal(back, finite)


def test_known_codes():
    # From the format definition: 1.0 = 0 0111 000, 448 = 0 1111 110,
    # 2^-6 = 0 0001 000 (smallest normal), 2^-9 = 0 0000 001 (smallest subnormal).
    vals = np.array([1.0, 448.0, 2.0 ** -6, 2.0 ** -9, -1.0, -448.0], dtype=np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), [0x38, 0x7E, 0x08, 0x01, 0xB8, 0xFE])


def test_midpoints_round_to_even_code():
    mids = ((GRID[:-1] + GRID[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (GRID[:-1] + GRID[1:]) / 2)  # exact in fp32
    codes = oracle.e4m3_encode(mids)
    lo = np.arange(GRID.size - 1)
    expect = np.where(lo % 2 == 0, lo, lo + 1)
    np.testing.assert_array_equal(codes, expect.astype(np.uint8))
    # One fp32 ulp either side of a midpoint goes to the nearer neighbour.
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    np.testing.assert_array_equal(oracle.e4m3_encode(up), (lo + 1).astype(np.uint8))
    np.testing.assert_array_equal(oracle.e4m3_encode(dn), lo.astype(np.uint8))
    np.testing.assert_array_equal(oracle.e4m3_encode(-mids), expect.astype(np.uint8) | 0x80)


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_exhaustive_bf16_vs_bruteforce():
    f = np.clip(_all_finite_bf16(), -448.0, 448.0).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(f), bruteforce_e4m3(f))


def test_exhaustive_bf16_vs_torch_cast():
    f = np.clip(_all_finite_bf16(), -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(f), ref)


def test_random_fp32_vs_bruteforce():
    rng = np.random.default_rng(1234)
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)).astype(np.float32)
    sign = rng.choice([-1.0, 1.0], mags.size).astype(np.float32)
    v = mags * sign
    np.testing.assert_array_equal(oracle.e4m3_encode(v), bruteforce_e4m3(v))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


@pytest.mark.parametrize("v,code", [(449.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE), (464.0, 0x7E),
                                    (-0.0, 0x80), (0.0, 0x00), (-1e-6, 0x80), (1e-6, 0x00),
                                    (-(2.0 ** -10), 0x80), (2.0 ** -10 * 1.0000001, 0x01)])
def test_saturation_and_signed_zero(v, code):
    assert int(oracle.e4m3_encode(np.array([v], dtype=np.float32))[0]) == code
