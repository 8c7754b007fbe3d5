"""Host-side checks of the C ABI (no GPU needed).

* libtfq.so loads and exports every function include/tfq.h declares, and the
  binding declares the same set;
* argument validation rejects bad calls before touching the GPU;
* on a machine without a GPU a valid call fails loudly (TFQ_ECUDA), it never
  falls back to anything.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from int8_w8a8_quantized_b200 import _capi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tfq.h")


def _declared():
    src = open(HEADER, encoding="utf-8").read()
    return re.findall(r"TFQ_API\s+[\w\s\*]+?\b(tfq_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _capi.load_library()


def test_header_declarations_match_binding():
    names = _declared()
    assert len(names) == len(set(names)) and names
    assert set(names) == set(_capi.SIGNATURES)


def test_header_limits_match_binding():
    text = open(os.path.join(ROOT, "include", "tfq.h"), encoding="utf-8").read()
    assert re.search(r"#define TFQ_INT8_MAX_K (\d+)", text).group(1) == str(_capi.TFQ_INT8_MAX_K)
    assert re.search(r"#define TFQ_MULTI_MAX_LINEARS (\d+)", text).group(1) == str(_capi.TFQ_MULTI_MAX_LINEARS)
    assert re.search(r"#define TFQ_QUANT_MAX_K \(1 << (\d+)\)", text).group(1) == str(_capi.TFQ_QUANT_MAX_K.bit_length() - 1)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _capi.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    assert _capi.status_string(0) == "TFQ_OK"
    assert _capi.status_string(4) == "TFQ_ETIMEOUT"
    assert _capi.status_string(99) == "unknown"
    assert lib.tfq_version() == 101


ALIGNED = 0x10000  # a fake, 16-byte aligned address: never dereferenced by a rejected call


@pytest.mark.parametrize("args,status", [
    ((ALIGNED, 4, 24, 448.0, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),        # K % 16
    ((ALIGNED, 4, 32, 500.0, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),        # qmax > 448
    ((ALIGNED, 4, 32, 0.5, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),          # qmax < 1
    ((ALIGNED, 4, 32, float("nan"), ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),
    ((None, 4, 32, 448.0, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),           # null x
    ((ALIGNED, 4, 32, 448.0, ALIGNED, None, None), _capi.TFQ_EINVAL),           # null s
    ((ALIGNED + 8, 4, 32, 448.0, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),    # misaligned
    ((ALIGNED, -1, 32, 448.0, ALIGNED, ALIGNED, None), _capi.TFQ_EINVAL),
    ((ALIGNED, 4, (1 << 24) + 16, 448.0, ALIGNED, ALIGNED, None), _capi.TFQ_EUNSUPPORTED),
    ((ALIGNED, 0, 32, 448.0, None, None, None), _capi.TFQ_OK),                  # M == 0: no-op
])
def test_quant_act_validation(lib, args, status):
    assert lib.tfq_quant_act_fp8_per_token(*args) == status
    if status != _capi.TFQ_OK:
        assert _capi.last_error_message()


def test_quant_weight_validation(lib):
    f = lib.tfq_quant_weight_per_channel
    assert f(ALIGNED, 4, 32, 7, 448.0, ALIGNED, ALIGNED, None) == _capi.TFQ_EINVAL            # dtype
    assert f(ALIGNED, 4, 32, _capi.TFQ_DTYPE_INT8, 200.0, ALIGNED, ALIGNED, None) == _capi.TFQ_EINVAL
    assert f(ALIGNED, 4, 40, _capi.TFQ_DTYPE_FP8_E4M3, 448.0, ALIGNED, ALIGNED, None) == _capi.TFQ_EINVAL
    assert f(ALIGNED, 0, 32, _capi.TFQ_DTYPE_INT8, 127.0, None, None, None) == _capi.TFQ_OK


@pytest.mark.parametrize("M,N,K,status", [
    (4, 16, 24, _capi.TFQ_EINVAL),     # K % 16
    (4, 16, 0, _capi.TFQ_EINVAL),      # K == 0
    (4, 12, 32, _capi.TFQ_EINVAL),     # N % 8
    (-1, 16, 32, _capi.TFQ_EINVAL),
    (1 << 31, 16, 32, _capi.TFQ_EUNSUPPORTED),
    (0, 16, 32, _capi.TFQ_OK),         # empty: no-op
    (4, 0, 32, _capi.TFQ_OK),
])
@pytest.mark.parametrize("entry", ["tfq_scaled_fp8_linear", "tfq_scaled_fp8_linear_noalloc"])
def test_gemm_validation(lib, entry, M, N, K, status):
    f = getattr(lib, entry)
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, M, N, K, ALIGNED, None) == status


def test_int8_gemm_k_limit(lib):
    """The INT8 GEMM's s32 sum is exact only for K < TFQ_INT8_MAX_K (128^2 K < 2^31)."""
    f = lib.tfq_scaled_int8_linear
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 131072, ALIGNED, None) == _capi.TFQ_EUNSUPPORTED
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 0, 16, 131072, ALIGNED, None) == _capi.TFQ_EUNSUPPORTED
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 0, 16, 131056, ALIGNED, None) == _capi.TFQ_OK  # empty


@pytest.mark.parametrize("entry", ["tfq_scaled_fp8_linear", "tfq_scaled_fp8_linear_noalloc"])
def test_gemm_rejects_null_and_misaligned(lib, entry):
    f = getattr(lib, entry)
    assert f(None, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 32, ALIGNED, None) == _capi.TFQ_EINVAL
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED + 2, 4, 16, 32, ALIGNED, None) == _capi.TFQ_EINVAL
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 32, ALIGNED + 4, None) == _capi.TFQ_EINVAL


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly(lib):
    st = lib.tfq_quant_act_fp8_per_token(ALIGNED, 4, 32, 448.0, ALIGNED, ALIGNED, None)
    assert st in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)
    assert lib.tfq_scaled_fp8_linear(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 32, ALIGNED, None) \
        in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)
    assert lib.tfq_scaled_fp8_linear_noalloc(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 32, ALIGNED, None) \
        in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)


def test_wait_selftest_rejects_bad_limits_before_any_launch(lib):
    assert lib.tfq_selftest_wait_timeout(0, None) == _capi.TFQ_EINVAL
    assert lib.tfq_selftest_wait_timeout(10_000_001, None) == _capi.TFQ_EINVAL


def test_mxfp8_scale_bytes(lib):
    assert lib.tfq_mxfp8_scale_bytes(1, 32) == 512
    assert lib.tfq_mxfp8_scale_bytes(128, 128) == 512
    assert lib.tfq_mxfp8_scale_bytes(129, 160) == 2 * 2 * 512
    assert lib.tfq_mxfp8_scale_bytes(75600, 5120) == 591 * 40 * 512
    assert lib.tfq_mxfp8_scale_bytes(0, 64) == 0
    assert lib.tfq_mxfp8_scale_bytes(-1, 64) == -1


def test_mxfp8_validation(lib):
    q = lib.tfq_quant_mxfp8
    assert q(ALIGNED, 4, 48, ALIGNED, ALIGNED, None) == _capi.TFQ_EINVAL          # K % 32
    assert q(ALIGNED, -1, 64, ALIGNED, ALIGNED, None) == _capi.TFQ_EINVAL
    assert q(ALIGNED, 4, 64, ALIGNED, None, None) == _capi.TFQ_EINVAL             # null sf
    assert q(ALIGNED, 4, 64, ALIGNED, ALIGNED + 4, None) == _capi.TFQ_EINVAL      # misaligned sf
    assert q(ALIGNED, 4, (1 << 24) + 32, ALIGNED, ALIGNED, None) == _capi.TFQ_EUNSUPPORTED
    assert q(None, 0, 64, None, None, None) == _capi.TFQ_OK                       # empty: no-op
    g = lib.tfq_mxfp8_linear
    assert g(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 48, ALIGNED, None) == _capi.TFQ_EINVAL  # K % 32
    assert g(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 12, 64, ALIGNED, None) == _capi.TFQ_EINVAL  # N % 8
    assert g(ALIGNED, None, ALIGNED, ALIGNED, None, 4, 16, 64, ALIGNED, None) == _capi.TFQ_EINVAL     # null sf_a
    assert g(ALIGNED, ALIGNED, ALIGNED, ALIGNED + 8, None, 4, 16, 64, ALIGNED, None) == _capi.TFQ_EINVAL
    assert g(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 0, 16, 64, ALIGNED, None) == _capi.TFQ_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_mxfp8_valid_call_without_gpu_fails_loudly(lib):
    assert lib.tfq_quant_mxfp8(ALIGNED, 4, 64, ALIGNED, ALIGNED, None) in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)
    assert lib.tfq_mxfp8_linear(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, 4, 16, 64, ALIGNED, None) \
        in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)


def test_missing_library_raises_no_fallback():
    """Without libtfq.so every call raises: there is no other implementation
    to fall back to.  Run in a fresh process (the loaded library is cached)."""
    import sys
    code = ("from int8_w8a8_quantized_b200 import _capi\n"
            "_capi.LIB_PATH = '/nonexistent/libtfq.so'\n"
            "import int8_w8a8_quantized_b200 as p\n"
            "try:\n"
            "    p.raw.tfq_version()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.startswith("raised:") and "not built" in r.stdout


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "tfq.h"

int main(void)
{
    const void *p = (const void *)0x10000; /* aligned, never dereferenced: every call below is rejected */
    if (tfq_version() != 101)
        return 1;
    if (strcmp(tfq_status_string(TFQ_EINVAL), "TFQ_EINVAL") != 0)
        return 2;
    if (tfq_quant_act_fp8_per_token(p, 4, 24, 448.0f, (void *)p, (float *)p, NULL) != TFQ_EINVAL)
        return 3;
    if (tfq_last_error_message()[0] == '\0')
        return 4;
    if (tfq_scaled_fp8_linear(p, (const float *)p, p, (const float *)p, NULL, 4, 12, 32, (void *)p, NULL)
        != TFQ_EINVAL)
        return 5;
    if (tfq_mxfp8_scale_bytes(129, 160) != 2 * 2 * 512)
        return 6;
    if (tfq_selftest_wait_timeout(0, NULL) != TFQ_EINVAL)
        return 7;
    printf("ok\n");
    return 0;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/tfq.h compiles as strict C99 (warnings as errors) and a C
    program links libtfq.so and gets the documented host-side answers."""
    src = tmp_path / "use_tfq.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_tfq"
    pkg = os.path.dirname(_capi.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", pkg, "-ltfq", f"-Wl,-rpath,{pkg}", "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_smoke_without_gpu_raises(lib):
    import __graft_entry__
    with pytest.raises(RuntimeError, match="CUDA device"):
        __graft_entry__.smoke()


def test_quant_scaled_linear_workspace_bytes(lib):
    """Two 128-byte lines of counters (the next row to quantize) plus one word
    per 128-row share of M, in whole 256-byte blocks."""
    f = lib.tfq_quant_scaled_fp8_linear_workspace_bytes
    for M in (1, 128, 129, 512, 6889, 75600, (1 << 31) - 1):
        n = f(M)
        assert n % 256 == 0 and n >= 4 * (32 + (M + 127) // 128) and n < 4 * (32 + (M + 127) // 128) + 256
    assert f(0) == 256 and f(-1) == 0


def _fused(lib, x=ALIGNED, M=1024, K=256, qmax=448.0, W=ALIGNED, sw=ALIGNED, b=None, N=256, A=ALIGNED,
           sa=ALIGNED, out=ALIGNED, ws=ALIGNED):
    return lib.tfq_quant_scaled_fp8_linear(x, M, K, qmax, W, sw, b, N, A, sa, out, ws, None)


def test_quant_scaled_linear_validation(lib):
    """The fused entry point checks the quantizer's and the GEMM's arguments
    and its workspace on the host, before any device work."""
    assert _fused(lib, K=24) == _capi.TFQ_EINVAL                      # K % 16
    assert _fused(lib, qmax=449.0) == _capi.TFQ_EINVAL
    assert _fused(lib, qmax=0.5) == _capi.TFQ_EINVAL
    assert _fused(lib, N=12) == _capi.TFQ_EINVAL                      # N % 8
    assert _fused(lib, x=None) == _capi.TFQ_EINVAL
    assert _fused(lib, W=None) == _capi.TFQ_EINVAL
    assert _fused(lib, sa=ALIGNED + 4) == _capi.TFQ_EINVAL
    assert _fused(lib, out=ALIGNED + 2) == _capi.TFQ_EINVAL
    assert _fused(lib, b=ALIGNED + 8) == _capi.TFQ_EINVAL
    assert _fused(lib, ws=None) == _capi.TFQ_EINVAL
    assert _fused(lib, ws=ALIGNED + 4) == _capi.TFQ_EINVAL
    assert _fused(lib, M=-1) == _capi.TFQ_EINVAL
    assert _fused(lib, M=1 << 31) == _capi.TFQ_EUNSUPPORTED
    assert _fused(lib, M=0, x=None, W=None, sw=None, A=None, sa=None, out=None, ws=None) == _capi.TFQ_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_quant_scaled_linear_without_gpu_fails_loudly(lib):
    assert _fused(lib) in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)


MULTI_ENTRIES = ("tfq_scaled_fp8_linear_multi", "tfq_scaled_int8_linear_multi")


def _multi(lib, n=3, M=1024, K=256, W=None, sw=None, b=None, N=None, out=None, A=ALIGNED, sa=ALIGNED,
           entry="tfq_scaled_fp8_linear_multi"):
    W = [ALIGNED] * n if W is None else W
    sw = [ALIGNED] * n if sw is None else sw
    N = [256] * n if N is None else N
    out = [ALIGNED] * n if out is None else out
    arr = _capi.pointer_array
    return getattr(lib, entry)(A, sa, M, K, n, arr(W) if W != "null" else None, arr(sw),
                               None if b is None else arr(b), (ctypes.c_int64 * len(N))(*N), arr(out), None)


@pytest.mark.parametrize("entry", MULTI_ENTRIES)
def test_multi_linear_validation(lib, entry):
    """The multi-Linear GEMMs check n, their arrays and every Linear's
    arguments on the host, before any device work."""
    def multi(**kw):
        return _multi(lib, entry=entry, **kw)
    assert multi(n=0, W=[], sw=[], N=[], out=[]) == _capi.TFQ_EINVAL
    assert multi(n=5) == _capi.TFQ_EINVAL
    assert multi(W="null") == _capi.TFQ_EINVAL
    assert multi(N=[256, 12, 256]) == _capi.TFQ_EINVAL                      # N % 8
    assert multi(W=[ALIGNED, None, ALIGNED]) == _capi.TFQ_EINVAL             # a null weight
    assert multi(out=[ALIGNED, ALIGNED, ALIGNED + 2]) == _capi.TFQ_EINVAL    # misaligned output
    assert multi(b=[None, ALIGNED + 8, None]) == _capi.TFQ_EINVAL            # misaligned bias
    assert multi(K=24) == _capi.TFQ_EINVAL
    assert multi(M=0, A=None, sa=None) == _capi.TFQ_OK                       # empty: no-op


def test_int8_multi_k_limit(lib):
    """Like tfq_scaled_int8_linear, the multi form refuses K whose s32 sum
    could overflow, before any device work."""
    K = _capi.TFQ_INT8_MAX_K
    assert _multi(lib, K=K, entry="tfq_scaled_int8_linear_multi") == _capi.TFQ_EUNSUPPORTED
    assert _multi(lib, K=K, M=0, A=None, sa=None, entry="tfq_scaled_int8_linear_multi") == _capi.TFQ_EUNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
@pytest.mark.parametrize("entry", MULTI_ENTRIES)
def test_multi_linear_without_gpu_fails_loudly(lib, entry):
    assert _multi(lib, entry=entry) in (_capi.TFQ_ECUDA, _capi.TFQ_EUNSUPPORTED)
