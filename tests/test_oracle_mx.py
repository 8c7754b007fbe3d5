"""Pins of the MXFP8 oracle (32-value blocks, E8M0 scales; the format named on
the TeleFuser "Quantization" page, section "Offline conversion", converted as
the OCP MX v1.0 specification describes): hand-worked blocks, the property
that fixes the shared exponent (the block maximum lands in [256, 512) before
saturation), a library cross-check of the element encoding, power-of-two
equivariance, the error bound, and the block-scaled GEMM against exact
rational brute force and against the pinned per-row GEMM with unit scales."""
import os
from fractions import Fraction

import numpy as np
import torch

import oracle
from tests._pins import bf16_bits, bits_to_f32, e4m3_spacing

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mx_blocks.txt")


def _load_blocks():
    out = []
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, code, xs, cs = [p.strip() for p in line.split("|")]
        x = np.zeros(32)
        q = np.zeros(32, dtype=np.uint8)
        for item in xs.split():
            i, v = item.split(":")
            val = float.fromhex(v) if v.startswith(("0x", "-0x")) else float(v)
            if i == "all":
                x[:] = val
            else:
                x[int(i)] = val
        for item in cs.split():
            i, c = item.split(":")
            if i == "all":
                q[:] = int(c, 16)
            else:
                q[int(i)] = int(c, 16)
        out.append((name, int(code), x, q))
    return out


def _bf16(x):
    t = torch.tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16)
    assert torch.equal(t.double(), torch.tensor(np.asarray(x, dtype=np.float64))), "value not exact in bf16"
    return bf16_bits(t)


def test_hand_blocks():
    blocks = _load_blocks()
    assert len(blocks) == 9
    for name, code, x, q in blocks:
        qo, sfo = oracle.quant_mxfp8(_bf16(x)[None, :])
        assert sfo[0, 0] == code, (name, sfo[0, 0], code)
        np.testing.assert_array_equal(qo[0], q, err_msg=name)


def _random_blocks(R, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, K, generator=g) * torch.exp2(torch.randint(-40, 41, (R, 1), generator=g).float())
    x[:, ::7] *= 30.0                                       # outliers inside blocks
    x[0] = 0.0                                              # all-zero blocks
    x[1, :32] = -0.0
    return x.to(torch.bfloat16)


def test_exponent_puts_block_max_in_256_512():
    """Exactly one power of two 2^E maps amax into [256, 512); E = floor(log2
    amax) - 8 is that one.  Where no clamp of E applies, the scaled maximum
    must land there, so its code is 0x78..0x7E (0x7E also for 448..512)."""
    x = _random_blocks(64, 256, seed=1)
    q, sf = oracle.quant_mxfp8(bf16_bits(x))
    xf = x.float().numpy().reshape(64, 8, 32)
    amax = np.abs(xf).max(axis=2)
    scaled = amax / np.exp2(sf.astype(np.float64) - 127)
    live = amax > 0
    assert np.all((scaled[live] >= 256) & (scaled[live] < 512))
    qb = q.reshape(64, 8, 32)
    arg = np.abs(xf).argmax(axis=2)
    top = np.take_along_axis(qb, arg[..., None], axis=2)[..., 0] & 0x7F
    assert np.all((top[live] >= 0x78) & (top[live] <= 0x7E))
    assert np.all(sf[~live] == 0)


def test_elements_match_torch_cast():
    """Given the scale, each element is torch's E4M3FN cast (round to nearest
    even) of x / 2^E after the clamp to +-448: a library cross-check of the
    element encoding."""
    x = _random_blocks(48, 512, seed=2)
    q, sf = oracle.quant_mxfp8(bf16_bits(x))
    scale = torch.tensor(np.exp2(sf.astype(np.float64) - 127)).repeat_interleave(32, dim=1)
    t = (x.double() / scale).clamp(-448.0, 448.0).float()
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q, ref)


def test_power_of_two_equivariance():
    """x * 2^j has the same codes and scale codes shifted by j (no clamping)."""
    x = _random_blocks(32, 256, seed=3)[2:]
    q0, sf0 = oracle.quant_mxfp8(bf16_bits(x))
    for j in (-5, 1, 17):
        q1, sf1 = oracle.quant_mxfp8(bf16_bits((x.double() * 2.0 ** j).to(torch.bfloat16)))
        np.testing.assert_array_equal(q1, q0)
        np.testing.assert_array_equal(sf1.astype(int), sf0.astype(int) + j)


def test_dequantization_error_bound():
    x = _random_blocks(40, 384, seed=4)
    q, sf = oracle.quant_mxfp8(bf16_bits(x))
    xf = x.double().numpy()
    scale = np.repeat(np.exp2(sf.astype(np.float64) - 127), 32, axis=1)
    deq = oracle.e4m3_decode(q) * scale
    t = np.abs(xf) / scale
    unsat = t <= 448.0
    err = np.abs(deq - xf)
    assert np.all(err[unsat] <= 0.5 * e4m3_spacing(np.minimum(t, 448.0))[unsat] * scale[unsat])
    assert np.all((q[~unsat] & 0x7F) == 0x7E)


def _frac_e4m3(code):
    v = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
    return Fraction(v)


def test_gemm_bruteforce_fraction():
    g = np.random.default_rng(5)
    M, N, K = 3, 4, 96
    A = g.integers(0, 0x7F, size=(M, K)).astype(np.uint8) | (g.integers(0, 2, size=(M, K)) << 7).astype(np.uint8)
    W = g.integers(0, 0x7F, size=(N, K)).astype(np.uint8) | (g.integers(0, 2, size=(N, K)) << 7).astype(np.uint8)
    sa = g.integers(100, 150, size=(M, K // 32)).astype(np.uint8)
    sw = g.integers(100, 150, size=(N, K // 32)).astype(np.uint8)
    bias = bf16_bits(torch.tensor([0.5, -1.25, 3.0, 0.0]).to(torch.bfloat16))
    y = oracle.mxfp8_linear(A, sa, W, sw, bias)
    bf = bits_to_f32(bias)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                b = k // 32
                acc += (_frac_e4m3(A[m, k]) * _frac_e4m3(W[n, k])
                        * Fraction(2) ** (int(sa[m, b]) - 127) * Fraction(2) ** (int(sw[n, b]) - 127))
            acc += Fraction(float(bf[n]))
            assert abs(Fraction(y[m, n]) - acc) <= abs(acc) * Fraction(1, 2 ** 50), (m, n)


def test_gemm_unit_scales_equal_per_row_gemm():
    """With every scale code 127 (2^0) the block-scaled GEMM is the per-row
    scaled GEMM with unit scales; moving one block's scale code by +1 doubles
    exactly that block's contribution."""
    g = np.random.default_rng(6)
    M, N, K = 5, 6, 128
    A = g.integers(0, 0x7E, size=(M, K)).astype(np.uint8)
    W = (g.integers(0, 0x7E, size=(N, K)) | 0x80).astype(np.uint8)
    one_a = np.full((M, K // 32), 127, np.uint8)
    one_w = np.full((N, K // 32), 127, np.uint8)
    y = oracle.mxfp8_linear(A, one_a, W, one_w)
    y_ref = oracle.scaled_fp8_linear(A, np.ones(M, np.float32), W, np.ones(N, np.float32))
    np.testing.assert_array_equal(y, y_ref)
    sa = one_a.copy()
    sa[2, 1] = 128
    y2 = oracle.mxfp8_linear(A, sa, W, one_w)
    A_blk = np.zeros_like(A)
    A_blk[:, 32:64] = A[:, 32:64]
    block = oracle.scaled_fp8_linear(A_blk, np.ones(M, np.float32), W, np.ones(N, np.float32))
    expect = y.copy()
    expect[2] += block[2]
    np.testing.assert_array_equal(y2, expect)
