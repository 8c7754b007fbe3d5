"""The seeded input generators follow their stated recipes (CPU only):
determinism per seed, outlier columns, zero rows, heavy tails, weight
scale, the workloads' sizes and FLOP counts, and independence from both
sides of the comparison (no oracle, no CUDA binding)."""
import os
import re

import pytest
import torch

from int8_w8a8_quantized_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_same_seed_same_bits_other_seed_other_bits():
    a = workloads.activations(64, 256, seed=5, nu=3, amplitude=4.0, outlier_cols=3, outlier_mult=30.0,
                              zero_rows=2)
    b = workloads.activations(64, 256, seed=5, nu=3, amplitude=4.0, outlier_cols=3, outlier_mult=30.0,
                              zero_rows=2)
    c = workloads.activations(64, 256, seed=6, nu=3, amplitude=4.0, outlier_cols=3, outlier_mult=30.0,
                              zero_rows=2)
    assert a.dtype == torch.bfloat16 and a.shape == (64, 256)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_outlier_columns_and_zero_rows():
    M, K, c, mult = 2048, 512, 5, 50.0
    x = workloads.activations(M, K, seed=11, outlier_cols=c, outlier_mult=mult, zero_rows=7).float()
    zero = (x == 0).all(dim=1)
    assert int(zero.sum()) == 7
    col_amax = x[~zero].abs().amax(dim=0)
    ranked = col_amax.sort(descending=True).values
    median = col_amax.median()
    # N(0,1) columns of 2041 rows peak near 3.5; the c scaled ones near 50x that
    assert torch.all(ranked[:c] > 0.3 * mult * median)
    assert torch.all(ranked[c:] < 2.0 * median)


def test_student_t_tails():
    x = workloads.activations(512, 1024, seed=3, nu=4).double()
    z = workloads.activations(512, 1024, seed=3).double()

    def kurtosis(t):
        t = t - t.mean()
        return float((t ** 4).mean() / (t ** 2).mean() ** 2)
    assert abs(kurtosis(z) - 3.0) < 0.1          # normal: 3
    assert kurtosis(x) > 5.0                      # Student-t, nu = 4: no finite fourth moment
    assert abs(float(x.var()) - 2.0) < 0.3        # variance nu / (nu - 2) = 2


def test_weight_and_bias_scale():
    w = workloads.weights(1024, 1024, seed=1, std=0.015).double()
    assert abs(float(w.std()) / 0.015 - 1.0) < 0.01 and abs(float(w.mean())) < 1e-4
    b = workloads.bias(4096, seed=2).double()
    assert abs(float(b.std()) / 0.01 - 1.0) < 0.05


def test_workload_sizes_and_flops():
    v, i, r = workloads.VIDEO_DIT, workloads.IMAGE_DIT, workloads.REDUCED_QMAX
    assert v.M == 21 * 45 * 80 and i.M == 83 * 83
    assert v.x_shapes() == {"x_attn": 5120, "x_o": 5120, "x_ffn": 5120, "x_ffn_h": 13824}
    assert v.flops() == 2 * 75600 * (4 * 5120 * 5120 + 2 * 5120 * 13824)
    assert i.flops() == 2 * 6889 * (4 * 3072 * 3072 + 2 * 3072 * 12288)
    assert r.flops() == 2 * 2 * 32760 * 13824 * 5120      # two activation qmaxes, 7 and 14
    for wl in workloads.WORKLOADS.values():
        for lin in wl.linears:
            assert lin.K % 16 == 0 and lin.N % 8 == 0    # the GEMM's size contract


def test_quantizer_input_recipe():
    x = workloads.quantizer_input().float()
    assert x.shape == (8192, 3072)
    zero = (x == 0).all(dim=1)
    assert int(zero.sum()) == 16
    col_amax = x[~zero].abs().amax(dim=0)
    assert int((col_amax > 10 * col_amax.median()).sum()) == round(0.01 * 3072)


def test_generators_hold_no_method_code():
    src = open(os.path.join(ROOT, "int8_w8a8_quantized_b200", "workloads.py"), encoding="utf-8").read()
    assert not re.search(r"^\s*(from|import)\s+(oracle|\.?_capi|int8_w8a8_quantized_b200\._capi)", src, re.M)
    assert "float8" not in src and "e4m3" not in src.lower()     # no casts to the quantized formats
