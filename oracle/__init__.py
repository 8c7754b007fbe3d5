"""CPU oracle for the W8A8 scaled-FP8 Linear -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package.  The product (the CUDA library
``libtfq.so`` and the ``int8_w8a8_quantized_b200`` binding) never imports it,
and the two share no code.

The arithmetic lives in ``tfq_oracle.c`` (plain C, IEEE fp32 divisions, an
explicit E4M3FN encoder written from the format definition, a double
accumulated GEMM).  This module only compiles it with gcc when needed and
marshals numpy arrays through ctypes.

What each function follows (page titles and sections of the source pages):

* ``quant_rows_fp8``: TeleFuser "Quantization", "Scaled FP8 checkpoints:
  W8A8" (s = max|x| / max(E4M3FN), q = cast(clamp(x/s))); the reduced qmax
  (14, 7) of LightX2V "模型量化技术", "MiniMax-H3 FP8 FP16 累加".
* ``quant_rows_int8``: TeleFuser "Quantization", "Core ideas" (s = max|x|/127,
  q = clamp(round(x/s), -128, 127)), one scale per output row ("Offline
  conversion").
* ``scaled_fp8_linear``: TeleFuser "Quantization", "Scaled FP8 checkpoints"
  and "tf-kernel FP8: online W8A8" (per-token x per-output-channel scaled
  GEMM with BF16 output); computed here in double, not rounded.
* ``scaled_int8_linear``: the INT8 W8A8 modes of LightX2V "模型量化技术",
  quantization-mode table (INT8 per-channel weights, dynamic per-token INT8
  activations), exact int64 sums.
* ``fp8_block_prefix_sums``: the running sums of the FP8 GEMM at every
  32-element block of K (their final value and largest magnitude), for the
  FP16-accumulator study of LightX2V "模型量化技术", "MiniMax-H3 FP8 FP16
  累加" (FP16 partial sums overflow at qmax 14 and 12, not at 7).
* ``quant_mxfp8`` / ``mxfp8_linear``: MXFP8 as named on the TeleFuser
  "Quantization" page, "Offline conversion" (32-value blocks, E8M0 scales),
  with the conversion of the OCP Microscaling (MX) v1.0 specification; the
  GEMM applies both block scales per 32-element block of K, in double.

Every function is pinned by the ``-m "not gpu"`` tests against values fixed
by the format definition, brute force and invariants (see ``tests/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tfq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-fexcess-precision=standard",
           "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``tfq_oracle.c`` into ``liboracle.so`` (gcc), if stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # TFQ_ORACLE_LIB names another build of tfq_oracle.c to load
            # instead: the mutation test runs the pins against copies of the
            # source with a planted mistake this way.  Taking it is announced
            # on stderr, and the GPU parity tests refuse to run under it
            # (tests/conftest.py), so a stray variable cannot swap the checker
            # silently.
            override = os.environ.get("TFQ_ORACLE_LIB")
            if override:
                sys.stderr.write(f"oracle: loading {override} (named by TFQ_ORACLE_LIB) "
                                 "instead of the built oracle\n")
            lib = ctypes.CDLL(override if override else build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.tfq_oracle_e4m3_decode.restype = ctypes.c_double
            lib.tfq_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.tfq_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.tfq_oracle_e4m3_encode.argtypes = [ctypes.c_float]
            for name in ("tfq_oracle_quant_rows_fp8", "tfq_oracle_quant_rows_int8"):
                fn = getattr(lib, name)
                fn.restype = None
                fn.argtypes = [P, I64, I64, ctypes.c_float, P, P]
            for name in ("tfq_oracle_scaled_fp8_linear", "tfq_oracle_scaled_int8_linear"):
                fn = getattr(lib, name)
                fn.restype = None
                fn.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P]
            lib.tfq_oracle_fp8_block_prefix_sums.restype = None
            lib.tfq_oracle_fp8_block_prefix_sums.argtypes = [P, P, I64, I64, I64, I64, P, I64, P, P]
            lib.tfq_oracle_quant_mxfp8.restype = None
            lib.tfq_oracle_quant_mxfp8.argtypes = [P, I64, I64, P, P]
            lib.tfq_oracle_mxfp8_linear.restype = None
            lib.tfq_oracle_mxfp8_linear.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P]
            lib.tfq_oracle_num_threads.restype = ctypes.c_int
            lib.tfq_oracle_num_threads.argtypes = []
            lib.tfq_oracle_set_num_threads.restype = None
            lib.tfq_oracle_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().tfq_oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().tfq_oracle_set_num_threads(int(n))


def e4m3_decode(codes) -> np.ndarray:
    """E4M3FN code bytes -> float64 values (NaN for S.1111.111)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    flat = c.reshape(-1)
    o = out.reshape(-1)
    for i in range(flat.size):
        o[i] = lib.tfq_oracle_e4m3_decode(int(flat[i]))
    return out


def e4m3_encode(values) -> np.ndarray:
    """float32 values -> E4M3FN codes (RNE, saturating at +-448)."""
    lib = _load()
    v = np.asarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    flat = v.reshape(-1)
    o = out.reshape(-1)
    for i in range(flat.size):
        o[i] = lib.tfq_oracle_e4m3_encode(float(flat[i]))
    return out


def _bf16_bits(x) -> np.ndarray:
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as their uint16 bit patterns")
    return a


def quant_rows_fp8(x_bits, qmax: float = 448.0):
    """Per-row FP8 quantization of bf16 bits [R, K] -> (codes u8 [R,K], s f32 [R])."""
    x = _bf16_bits(x_bits)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.uint8)
    s = np.empty((R,), dtype=np.float32)
    _load().tfq_oracle_quant_rows_fp8(_ptr(x), R, K, float(qmax), _ptr(q), _ptr(s))
    return q, s


def quant_rows_int8(x_bits, qmax: float = 127.0):
    """Per-row INT8 quantization of bf16 bits [R, K] -> (codes i8 [R,K], s f32 [R])."""
    x = _bf16_bits(x_bits)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.int8)
    s = np.empty((R,), dtype=np.float32)
    _load().tfq_oracle_quant_rows_int8(_ptr(x), R, K, float(qmax), _ptr(q), _ptr(s))
    return q, s


def _linear(fn, A, s_a, W, s_w, bias_bits, rows, code_dtype):
    A = np.ascontiguousarray(A, dtype=code_dtype)
    W = np.ascontiguousarray(W, dtype=code_dtype)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = A.shape
    N, K2 = W.shape
    if K2 != K or s_a.shape != (M,) or s_w.shape != (N,):
        raise ValueError("shape mismatch")
    b = None
    if bias_bits is not None:
        b = _bf16_bits(bias_bits)
        if b.shape != (N,):
            raise ValueError("bias shape")
    r = None
    nrows = M
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        if r.size and (r.min() < 0 or r.max() >= M):
            raise ValueError("row index out of range")
        nrows = r.size
    y = np.empty((nrows, N), dtype=np.float64)
    fn(_ptr(A), _ptr(s_a), _ptr(W), _ptr(s_w), _ptr(b), M, N, K, _ptr(r), nrows, _ptr(y))
    return y


def scaled_fp8_linear(A, s_a, W, s_w, bias_bits=None, rows=None) -> np.ndarray:
    """y[i,n] = sum_k dec(A[m,k]) dec(W[n,k]) * s_a[m] * s_w[n] + bias[n] (double)."""
    return _linear(_load().tfq_oracle_scaled_fp8_linear, A, s_a, W, s_w,
                   bias_bits, rows, np.uint8)


def scaled_int8_linear(A, s_a, W, s_w, bias_bits=None, rows=None) -> np.ndarray:
    """y[i,n] = sum_k A[m,k] W[n,k] * s_a[m] * s_w[n] + bias[n] (double)."""
    return _linear(_load().tfq_oracle_scaled_int8_linear, A, s_a, W, s_w,
                   bias_bits, rows, np.int8)


def fp8_block_prefix_sums(A, W, block: int = 32, rows=None):
    """The FP8 GEMM's running sums at every `block`-element boundary of K:
    (final [rows, N] = sum_k dec(A) dec(W), prefix_max [rows, N] = the largest
    |running sum| at a block boundary), exact, no scales or bias.  For the
    FP16-accumulator study of LightX2V "模型量化技术", "MiniMax-H3 FP8 FP16
    累加"."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    W = np.ascontiguousarray(W, dtype=np.uint8)
    M, K = A.shape
    N, K2 = W.shape
    if K2 != K or block < 1:
        raise ValueError("shape mismatch")
    r = None
    nrows = M
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        if r.size and (r.min() < 0 or r.max() >= M):
            raise ValueError("row index out of range")
        nrows = r.size
    final = np.empty((nrows, N), dtype=np.float64)
    pmax = np.empty((nrows, N), dtype=np.float64)
    _load().tfq_oracle_fp8_block_prefix_sums(_ptr(A), _ptr(W), M, N, K, int(block), _ptr(r), nrows, _ptr(final),
                                             _ptr(pmax))
    return final, pmax


def quant_mxfp8(x_bits):
    """MXFP8 quantization of bf16 bits [R, K] (K % 32 == 0) ->
    (codes u8 [R, K], E8M0 scale codes u8 [R, K // 32], row-major)."""
    x = _bf16_bits(x_bits)
    R, K = x.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q = np.empty((R, K), dtype=np.uint8)
    sf = np.empty((R, K // 32), dtype=np.uint8)
    _load().tfq_oracle_quant_mxfp8(_ptr(x), R, K, _ptr(q), _ptr(sf))
    return q, sf


def mxfp8_linear(A, sf_a, W, sf_w, bias_bits=None, rows=None) -> np.ndarray:
    """y[i,n] = sum_b 2^(sf_a[m,b]-127) 2^(sf_w[n,b]-127) sum_{k in b} dec(A) dec(W)
    + bias[n] (double); sf_* are row-major [rows, K // 32] E8M0 codes."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    W = np.ascontiguousarray(W, dtype=np.uint8)
    sf_a = np.ascontiguousarray(sf_a, dtype=np.uint8)
    sf_w = np.ascontiguousarray(sf_w, dtype=np.uint8)
    M, K = A.shape
    N, K2 = W.shape
    if K2 != K or K % 32 or sf_a.shape != (M, K // 32) or sf_w.shape != (N, K // 32):
        raise ValueError("shape mismatch")
    b = None
    if bias_bits is not None:
        b = _bf16_bits(bias_bits)
        if b.shape != (N,):
            raise ValueError("bias shape")
    r = None
    nrows = M
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        if r.size and (r.min() < 0 or r.max() >= M):
            raise ValueError("row index out of range")
        nrows = r.size
    y = np.empty((nrows, N), dtype=np.float64)
    _load().tfq_oracle_mxfp8_linear(_ptr(A), _ptr(sf_a), _ptr(W), _ptr(sf_w), _ptr(b), M, N, K, _ptr(r),
                                    nrows, _ptr(y))
    return y
