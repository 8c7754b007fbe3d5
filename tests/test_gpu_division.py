"""The quantizers' branch-free division (a two-term reciprocal of the row
scale and one Markstein correction) against CUDA's IEEE division __fdiv_rn,
bit for bit, through the tfq_selftest_div_rn self-check entry point: every
finite bf16 numerator against row scales s = fl32(amax / qmax) drawn over
the whole range the quantizers take this path for (the 1e-12 floor up to
2^64; larger scales use the IEEE division), plus scales next to powers of
two and random fp32 numerators.  Quotients below 2^-58 in magnitude, far
below every code's rounding threshold, need only be tiny with the sign of
the numerator."""

import numpy as np
import pytest
import torch

from int8_w8a8_quantized_b200 import _capi
from tests import _gpu

pytestmark = pytest.mark.gpu

# Largest row scale the quantizers divide by without __fdiv_rn.
DIV_MAX_SCALE = np.float32(2.0 ** 64)


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def _run(a: np.ndarray, b: np.ndarray):
    ta = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    tb = torch.from_numpy(np.ascontiguousarray(b, dtype=np.float32)).cuda()
    ours = torch.empty_like(ta)
    ieee = torch.empty_like(ta)
    st = _capi.raw.tfq_selftest_div_rn(ta.data_ptr(), tb.data_ptr(), ta.numel(), ours.data_ptr(),
                                       ieee.data_ptr(), _gpu.stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    torch.cuda.synchronize()
    o = ours.cpu().numpy()
    r = ieee.cpu().numpy()
    exact = np.abs(a.astype(np.float64) / b.astype(np.float64)) >= 2.0 ** -58
    bad = np.nonzero(exact & (o.view(np.uint32) != r.view(np.uint32)))[0]
    assert bad.size == 0, (f"{bad.size} mismatches; first a={a[bad[0]]!r} b={b[bad[0]]!r} "
                           f"ours={o[bad[0]]!r} ieee={r[bad[0]]!r}")
    # tiny quotients: both tiny (so both encode to +-0) with the sign of a
    tiny = ~exact
    assert np.all(np.abs(o[tiny]) < 2.0 ** -53) and np.all(np.abs(r[tiny]) < 2.0 ** -53)
    assert np.array_equal(np.signbit(o[tiny]), np.signbit(a[tiny]))
    assert np.array_equal(np.signbit(r[tiny]), np.signbit(a[tiny]))
    return int(exact.sum())


def _scales(rng, n):
    qmax = rng.choice(np.array([448.0, 14.0, 7.0, 127.0, 21.0, 100.0, 1.0], dtype=np.float32), n)
    amax = np.exp(rng.uniform(np.log(1e-12), np.log(3e38), n)).astype(np.float32)
    amax[: n // 8] = np.float32(1e-12)                    # the floor
    s = (np.maximum(amax, np.float32(1e-12)) / qmax).astype(np.float32)
    s = np.minimum(s, DIV_MAX_SCALE)                      # larger scales use the IEEE division
    # scales just around powers of two and their neighbours
    p2 = (2.0 ** rng.integers(-40, 64, n // 4)).astype(np.float32)
    s2 = np.concatenate([p2, np.nextafter(p2, np.float32(0)), np.nextafter(p2, np.float32(np.inf))])
    return np.concatenate([s, s2]).astype(np.float32)


def test_all_bf16_numerators_many_scales():
    _gpu.lib()
    rng = np.random.default_rng(2024)
    a_all = _all_finite_bf16()
    scales = _scales(rng, 1600)
    checked = 0
    for chunk in np.array_split(scales, 40):
        a = np.tile(a_all, chunk.size)
        b = np.repeat(chunk, a_all.size)
        keep = np.abs(a.astype(np.float64) / b.astype(np.float64)) <= 448.0 * 1.001
        checked += _run(a[keep], b[keep])
    assert checked > 10_000_000


def test_random_fp32_numerators():
    _gpu.lib()
    rng = np.random.default_rng(7)
    n = 4_000_000
    b = _scales(rng, n // 2)[: n]
    b = np.resize(b, n).astype(np.float32)
    t = rng.uniform(-448.0, 448.0, n)                     # target quotients
    a64 = t * b.astype(np.float64)
    keep = np.abs(a64) <= 3.0e38                          # finite fp32 numerators only
    a = a64[keep].astype(np.float32)
    b = b[keep]
    a[::7] = -a[::7]
    a[::11] = 0.0
    a[::13] = -0.0
    assert np.isfinite(a).all() and a.size > n // 2
    _run(a, b)
