"""The oracle's pins catch plausible mistakes in it (CPU only).

Each case plants one mistake in a copy of ``oracle/tfq_oracle.c``: a dropped
term, a wrong sign, index or constant, a transposed operand, another rounding
rule.  The copy is built with the oracle's own compiler flags, and the pin
tests (``tests/test_oracle_*.py``) run against it through
``TFQ_ORACLE_LIB``.  Every mutant must fail at least one pin.  The unmodified
copy, built and run the same way, must pass them all.

Left out: changes that cannot alter any result, e.g. the FP8 quantizer's
clamp to +-qmax (x/s exceeds qmax by at most one rounding, and the encoder
rounds that back to qmax) or the INT8 clamp at -128 (|x/s| rounds to at most
127).
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tfq_oracle.c")
PIN_FILES = ["tests/test_oracle_e4m3.py", "tests/test_oracle_quant.py",
             "tests/test_oracle_gemm.py", "tests/test_oracle_mx.py"]

# name -> [(text in tfq_oracle.c, replacement)]; each text occurs exactly once.
MUTANTS = {
    # block prefix sums (FP16-accumulator study)
    "block_prefix_signed_max": [("if (fabs(acc) > pmax)\n                        pmax = fabs(acc);",
                                 "if (acc > pmax)\n                        pmax = acc;")],
    "block_prefix_boundary_off_by_one": [("if ((k + 1) % block == 0 || k + 1 == K) {",
                                          "if (k % block == 0 || k + 1 == K) {")],
    "block_prefix_no_partial_last_block": [("if ((k + 1) % block == 0 || k + 1 == K) {",
                                            "if ((k + 1) % block == 0) {")],
    # E4M3FN decoding
    "decode_subnormal_exponent": [("mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);")],
    "decode_exponent_bias": [("ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 9)")],
    "decode_ignores_sign": [("    return sign ? -mag : mag;\n}", "    (void)sign;\n    return mag;\n}")],
    "decode_nan_whole_top_binade": [("if (e == 15 && m == 7)", "if (e == 15)")],
    # E4M3FN encoding
    "encode_ties_away": [("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;")],
    "encode_ties_down": [("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f;")],
    "encode_negative_zero_unsigned": [("signbit(t) ? 0x80 : 0x00", "(t < 0.0f) ? 0x80 : 0x00")],
    "encode_no_saturation": [("if (a > 448.0)\n        a = 448.0;", ""),
                             ("if (code > 0x7E)\n        code = 0x7E;", "")],
    "encode_subnormal_binade": [("if (e < -6)\n        e = -6;", "if (e < -7)\n        e = -7;")],
    "encode_log2_off_by_one": [("e = E - 1;          /* floor(log2(a)) */", "e = E;")],
    # per-row scale and quotient
    "scale_signed_max": [("float v = fabsf(bf16_bits_to_float(row[k]));", "float v = bf16_bits_to_float(row[k]);")],
    "scale_skips_last_element": [("    for (k = 0; k < K; ++k) {\n        float v = fabsf(bf16_bits_to_float(row[k]));",
                                  "    for (k = 0; k < K - 1; ++k) {\n        float v = fabsf(bf16_bits_to_float(row[k]));")],
    "scale_no_zero_floor": [("if (amax < 1e-12f)\n        amax = 1e-12f;", "")],
    "scale_by_reciprocal": [("return amax / qmax;", "return amax * (1.0f / qmax);")],
    "fp8_quotient_by_reciprocal": [
        ("float t = bf16_bits_to_float(row[k]) / sc;\n            if (t > qmax)",
         "float t = bf16_bits_to_float(row[k]) * (1.0f / sc);\n            if (t > qmax)")],
    "fp8_no_clamp": [("            if (t > qmax)\n                t = qmax;\n            if (t < -qmax)\n                t = -qmax;\n            q[r * K + k] = tfq_oracle_e4m3_encode(t);",
                      "            q[r * K + k] = tfq_oracle_e4m3_encode(t);")],
    "fp8_clamp_upper_only": [("            if (t < -qmax)\n                t = -qmax;\n            q[r * K + k] = tfq_oracle_e4m3_encode(t);",
                              "            q[r * K + k] = tfq_oracle_e4m3_encode(t);")],
    "int8_quotient_by_reciprocal": [
        ("float t = bf16_bits_to_float(row[k]) / sc;\n            double mag",
         "float t = bf16_bits_to_float(row[k]) * (1.0f / sc);\n            double mag")],
    "int8_round_half_away": [("double mag = round_half_even_nonneg(fabs((double)t));",
                              "double mag = floor(fabs((double)t) + 0.5);")],
    "int8_truncate": [("double mag = round_half_even_nonneg(fabs((double)t));",
                       "double mag = floor(fabs((double)t));")],
    # scaled FP8 GEMM
    "fp8_gemm_no_weight_scale": [("acc = acc * (double)s_a[m] * (double)s_w[n];", "acc = acc * (double)s_a[m];")],
    "fp8_gemm_weight_scale_index": [("acc = acc * (double)s_a[m] * (double)s_w[n];",
                                     "acc = acc * (double)s_a[m] * (double)s_w[m % N];")],
    "fp8_gemm_float_accumulator": [("            double acc = 0.0;\n            int64_t k;\n            for (k = 0; k < K; ++k)\n                acc += dec[a[k]] * dec[w[k]];",
                                    "            float acc = 0.0f;\n            int64_t k;\n            for (k = 0; k < K; ++k)\n                acc += (float)(dec[a[k]] * dec[w[k]]);")],
    "fp8_gemm_activation_scale_index": [("acc = acc * (double)s_a[m] * (double)s_w[n];",
                                         "acc = acc * (double)s_a[i] * (double)s_w[n];")],
    "fp8_gemm_drops_last_k": [("            for (k = 0; k < K; ++k)\n                acc += dec[a[k]] * dec[w[k]];",
                               "            for (k = 0; k < K - 1; ++k)\n                acc += dec[a[k]] * dec[w[k]];")],
    "fp8_gemm_bias_index": [("                acc += (double)bf16_bits_to_float(bias[n]);\n            y[i * N + n] = acc;\n        }\n    }\n}\n\n/*\n * INT8",
                             "                acc += (double)bf16_bits_to_float(bias[m % N]);\n            y[i * N + n] = acc;\n        }\n    }\n}\n\n/*\n * INT8")],
    "fp8_gemm_reversed_k": [("acc += dec[a[k]] * dec[w[k]];", "acc += dec[a[k]] * dec[w[K - 1 - k]];")],
    "fp8_gemm_no_bias": [("acc = acc * (double)s_a[m] * (double)s_w[n];\n            if (bias)\n",
                          "acc = acc * (double)s_a[m] * (double)s_w[n];\n            if (bias && 0)\n")],
    "fp8_gemm_bias_before_scales": [("            acc = acc * (double)s_a[m] * (double)s_w[n];\n            if (bias)\n                acc += (double)bf16_bits_to_float(bias[n]);\n            y[i * N + n] = acc;",
                                     "            if (bias)\n                acc += (double)bf16_bits_to_float(bias[n]);\n            acc = acc * (double)s_a[m] * (double)s_w[n];\n            y[i * N + n] = acc;")],
    "fp8_gemm_bias_subtracted": [("(double)s_w[n];\n            if (bias)\n                acc +=",
                                  "(double)s_w[n];\n            if (bias)\n                acc -=")],
    # scaled INT8 GEMM
    "int8_gemm_no_activation_scale": [("v = (double)acc * (double)s_a[m] * (double)s_w[n];",
                                       "v = (double)acc * (double)s_w[n];")],
    "int8_gemm_unsigned_activation": [("acc += (int64_t)a[k] * (int64_t)w[k];",
                                       "acc += (int64_t)(uint8_t)a[k] * (int64_t)w[k];")],
    "int8_gemm_drops_last_k": [("            for (k = 0; k < K; ++k)\n                acc += (int64_t)a[k] * (int64_t)w[k];",
                                "            for (k = 0; k < K - 1; ++k)\n                acc += (int64_t)a[k] * (int64_t)w[k];")],
    "int8_gemm_bias_subtracted": [("v += (double)bf16_bits_to_float(bias[n]);",
                                   "v -= (double)bf16_bits_to_float(bias[n]);")],
    # MXFP8 quantization
    "mx_emax_7": [("e = (E - 1) - 8;", "e = (E - 1) - 7;")],
    "mx_zero_block_unit_scale": [("if (amax == 0.0f)\n        return 0;", "if (amax == 0.0f)\n        return 127;")],
    "mx_exponent_floor_minus_126": [("if (e < -127)\n        e = -127;", "if (e < -126)\n        e = -126;")],
    "mx_scale_bias": [("scale = ldexp(1.0, (int)code - 127);", "scale = ldexp(1.0, (int)code - 126);")],
    "mx_block_max_skips_last": [("            for (k = 0; k < 32; ++k) {\n                float v = fabsf(bf16_bits_to_float(blk[k]));",
                                 "            for (k = 0; k < 31; ++k) {\n                float v = fabsf(bf16_bits_to_float(blk[k]));")],
    "mx_block_stride": [("const uint16_t *blk = x + r * K + b * 32;", "const uint16_t *blk = x + r * K + b * 16;")],
    "mx_element_scale_multiplied": [("double t = (double)bf16_bits_to_float(blk[k]) / scale;",
                                     "double t = (double)bf16_bits_to_float(blk[k]) * scale;")],
    "mx_signed_max": [("float v = fabsf(bf16_bits_to_float(blk[k]));", "float v = bf16_bits_to_float(blk[k]);")],
    # MXFP8 GEMM
    "mx_gemm_no_weight_scale": [("(int)sfa[m * nb + b] + (int)sfw[n * nb + b] - 254", "(int)sfa[m * nb + b] - 127")],
    "mx_gemm_first_block_scale": [("(int)sfw[n * nb + b]", "(int)sfw[n * nb]")],
    "mx_gemm_first_row_scale": [("(int)sfa[m * nb + b] + (int)sfw[n * nb + b]", "(int)sfa[b] + (int)sfw[n * nb + b]")],
    "mx_gemm_first_block_codes": [("const uint8_t *w = W + n * K + b * 32;", "const uint8_t *w = W + n * K;")],
    "mx_gemm_bias_subtracted": [("- 254);\n            }\n            if (bias)\n                acc +=",
                                 "- 254);\n            }\n            if (bias)\n                acc -=")],
}


def _mutate(src: str, edits) -> str:
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site not unique or gone: {old!r}"
        src = src.replace(old, new)
    return src


def _build_and_run(name: str, src: str, workdir: str):
    path = os.path.join(workdir, f"{name}.c")
    lib = os.path.join(workdir, f"lib{name}.so")
    with open(path, "w", encoding="utf-8") as fh:
        fh.write(src)
    cc = subprocess.run(["gcc", *oracle._CFLAGS, path, "-o", lib, "-lm"], capture_output=True, text=True)
    if cc.returncode != 0:
        return ("build", cc.stderr[-2000:])
    env = dict(os.environ, TFQ_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    run = subprocess.run([sys.executable, "-m", "pytest", *PIN_FILES, "-x", "-q", "-m", "not gpu",
                          "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    return (run.returncode, (run.stdout + run.stderr)[-2000:])


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    workdir = str(tmp_path_factory.mktemp("oracle_mutants"))
    base = open(SRC, encoding="utf-8").read()
    jobs = {"unmodified": base}
    jobs.update({name: _mutate(base, edits) for name, edits in MUTANTS.items()})
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        futures = {name: pool.submit(_build_and_run, name, src, workdir) for name, src in jobs.items()}
        return {name: f.result() for name, f in futures.items()}


def test_unmodified_copy_passes_every_pin(outcomes):
    rc, log = outcomes["unmodified"]
    assert rc == 0, log


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(outcomes, name):
    rc, log = outcomes[name]
    # pytest exits 1 when tests ran and some failed; anything else (a build
    # error, a collection error, a crash) does not show that a pin caught it
    assert rc == 1, f"{name}: exit {rc}\n{log}"
