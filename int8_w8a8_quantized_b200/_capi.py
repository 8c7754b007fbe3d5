"""ctypes binding of libtfq.so (include/tfq.h).

Two layers, both argument marshalling only (every step runs in the CUDA
library):

* ``raw``: the C functions with their C signatures (integers for pointers,
  a stream handle as an integer); the tests call the library through these;
* functions named like the C entry points that take torch CUDA tensors,
  check dtypes/shapes/devices, allocate outputs when none are given, pass
  ``data_ptr()`` and the current CUDA stream, and raise ``TfqError`` on a
  non-zero status.

There is no fallback: if libtfq.so is missing or cannot be loaded, every
call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libtfq.so")

TFQ_OK, TFQ_EINVAL, TFQ_EUNSUPPORTED, TFQ_ECUDA, TFQ_ETIMEOUT = range(5)
TFQ_DTYPE_FP8_E4M3, TFQ_DTYPE_INT8 = 0, 1
TFQ_QUANT_MAX_K = 1 << 24
TFQ_INT8_MAX_K = 131072  # the INT8 GEMM takes K < this (its s32 sum stays exact)
TFQ_MULTI_MAX_LINEARS = 4

# name -> (restype, argtypes), in the order include/tfq.h declares them
_P, _I64, _F, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
SIGNATURES = {
    "tfq_quant_act_fp8_per_token": (_I, [_P, _I64, _I64, _F, _P, _P, _P]),
    "tfq_quant_weight_per_channel": (_I, [_P, _I64, _I64, _I, _F, _P, _P, _P]),
    "tfq_scaled_fp8_linear": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "tfq_scaled_fp8_linear_multi": (_I, [_P, _P, _I64, _I64, _I, _P, _P, _P, _P, _P, _P]),
    "tfq_quant_scaled_fp8_linear_workspace_bytes": (ctypes.c_size_t, [_I64]),
    "tfq_quant_scaled_fp8_linear": (_I, [_P, _I64, _I64, _F, _P, _P, _P, _I64, _P, _P, _P, _P, _P]),
    "tfq_quant_act_int8_per_token": (_I, [_P, _I64, _I64, _F, _P, _P, _P]),
    "tfq_scaled_int8_linear": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "tfq_scaled_int8_linear_multi": (_I, [_P, _P, _I64, _I64, _I, _P, _P, _P, _P, _P, _P]),
    "tfq_scaled_fp8_linear_f16acc": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "tfq_mxfp8_scale_bytes": (_I64, [_I64, _I64]),
    "tfq_quant_mxfp8": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "tfq_mxfp8_linear": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "tfq_scaled_fp8_linear_noalloc": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "tfq_selftest_div_rn": (_I, [_P, _P, _I64, _P, _P, _P]),
    "tfq_selftest_wait_timeout": (_I, [ctypes.c_uint32, _P]),
    "tfq_device_error": (_I, [_P]),
    "tfq_status_string": (ctypes.c_char_p, [_I]),
    "tfq_last_error_message": (ctypes.c_char_p, []),
    "tfq_version": (_I, []),
}

_lock = threading.Lock()
_lib = None


class TfqError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {status_string(status)}: {message}")
        self.status = status


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Loads libtfq.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is not built; run `python -m int8_w8a8_quantized_b200.build`")
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


class _Raw:
    """The C entry points with their C signatures."""

    def __getattr__(self, name):
        if name not in SIGNATURES:
            raise AttributeError(name)
        return getattr(load_library(), name)


raw = _Raw()


def status_string(status: int) -> str:
    return load_library().tfq_status_string(int(status)).decode()


def last_error_message() -> str:
    return load_library().tfq_last_error_message().decode()


def _check(status: int, where: str) -> None:
    if status != TFQ_OK:
        raise TfqError(status, where, last_error_message())


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _require(t, dtype, ndim, name, device=None):
    """Checks a tensor argument: a contiguous CUDA tensor of `dtype` (an E4M3
    code tensor may also be torch.float8_e4m3fn: the same bytes) with `ndim`
    dimensions, on `device` when given (every operand of one call must live
    on one GPU)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    e4m3 = getattr(torch, "float8_e4m3fn", None)
    if t.dtype != dtype and not (dtype == torch.uint8 and e4m3 is not None and t.dtype == e4m3 and
                                 name in _E4M3_OPERANDS):
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {device}")


# Arguments that hold E4M3FN codes (uint8, or torch.float8_e4m3fn views of them).
_E4M3_OPERANDS = ("q", "A_q", "W_q")


def tfq_quant_act_fp8_per_token(x, qmax: float = 448.0, q=None, s=None, stream=None):
    """x bf16 [M, K] -> (q uint8 [M, K] E4M3FN codes, s fp32 [M])."""
    import torch
    _require(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty((M,), dtype=torch.float32, device=x.device)
    _require(q, torch.uint8, 2, "q", x.device)
    _require(s, torch.float32, 1, "s", x.device)
    if tuple(q.shape) != (M, K) or tuple(s.shape) != (M,):
        raise ValueError("output shapes do not match x")
    with torch.cuda.device(x.device):
        st = raw.tfq_quant_act_fp8_per_token(x.data_ptr(), M, K, float(qmax), q.data_ptr(), s.data_ptr(),
                                             _stream_handle(stream))
    _check(st, "tfq_quant_act_fp8_per_token")
    return q, s


def tfq_quant_weight_per_channel(w, dtype: str = "fp8", qmax: float | None = None, q=None, s=None, stream=None):
    """w bf16 [N, K] -> (codes [N, K] (uint8 E4M3FN or int8), s fp32 [N])."""
    import torch
    _require(w, torch.bfloat16, 2, "w")
    N, K = w.shape
    if dtype == "fp8":
        code, qdt, qmax = TFQ_DTYPE_FP8_E4M3, torch.uint8, 448.0 if qmax is None else qmax
    elif dtype == "int8":
        code, qdt, qmax = TFQ_DTYPE_INT8, torch.int8, 127.0 if qmax is None else qmax
    else:
        raise ValueError("dtype must be 'fp8' or 'int8'")
    if q is None:
        q = torch.empty((N, K), dtype=qdt, device=w.device)
    if s is None:
        s = torch.empty((N,), dtype=torch.float32, device=w.device)
    _require(q, qdt, 2, "q", w.device)
    _require(s, torch.float32, 1, "s", w.device)
    if tuple(q.shape) != (N, K) or tuple(s.shape) != (N,):
        raise ValueError("output shapes do not match w")
    with torch.cuda.device(w.device):
        st = raw.tfq_quant_weight_per_channel(w.data_ptr(), N, K, code, float(qmax), q.data_ptr(), s.data_ptr(),
                                              _stream_handle(stream))
    _check(st, "tfq_quant_weight_per_channel")
    return q, s


def tfq_scaled_fp8_linear(A_q, s_a, W_q, s_w, bias=None, out=None, stream=None):
    """A_q uint8 [M, K], s_a fp32 [M], W_q uint8 [N, K], s_w fp32 [N], bias bf16 [N] or None
    -> out bf16 [M, N]."""
    return _scaled_fp8_gemm("tfq_scaled_fp8_linear", A_q, s_a, W_q, s_w, bias, out, stream)


def tfq_scaled_fp8_linear_f16acc(A_q, s_a, W_q, s_w, bias=None, out=None, stream=None):
    """tfq_scaled_fp8_linear with FP16 partial sums on the tensor cores: the
    result is defined only while every partial sum fits in FP16, i.e. for
    activations quantized with a reduced qmax (7, 14)."""
    return _scaled_fp8_gemm("tfq_scaled_fp8_linear_f16acc", A_q, s_a, W_q, s_w, bias, out, stream)


def tfq_scaled_fp8_linear_noalloc(A_q, s_a, W_q, s_w, bias=None, out=None, stream=None):
    """tfq_scaled_fp8_linear that never allocates device memory (its kernel's
    scratch words live in a static array of the library)."""
    return _scaled_fp8_gemm("tfq_scaled_fp8_linear_noalloc", A_q, s_a, W_q, s_w, bias, out, stream)


def _scaled_fp8_gemm(entry, A_q, s_a, W_q, s_w, bias, out, stream):
    import torch
    _require(A_q, torch.uint8, 2, "A_q")
    dev = A_q.device
    _require(W_q, torch.uint8, 2, "W_q", dev)
    _require(s_a, torch.float32, 1, "s_a", dev)
    _require(s_w, torch.float32, 1, "s_w", dev)
    M, K = A_q.shape
    N, K2 = W_q.shape
    if K2 != K or s_a.shape[0] != M or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    if bias is not None:
        _require(bias, torch.bfloat16, 1, "bias", dev)
        if bias.shape[0] != N:
            raise ValueError("bias shape")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A_q.device)
    _require(out, torch.bfloat16, 2, "out", dev)
    if tuple(out.shape) != (M, N):
        raise ValueError("out shape")
    with torch.cuda.device(A_q.device):
        st = getattr(raw, entry)(A_q.data_ptr(), s_a.data_ptr(), W_q.data_ptr(), s_w.data_ptr(),
                                 None if bias is None else bias.data_ptr(), M, N, K, out.data_ptr(),
                                 _stream_handle(stream))
    _check(st, entry)
    return out


def tfq_quant_act_int8_per_token(x, qmax: float = 127.0, q=None, s=None, stream=None):
    """x bf16 [M, K] -> (q int8 [M, K], s fp32 [M]): dynamic per-token INT8."""
    import torch
    _require(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty((M,), dtype=torch.float32, device=x.device)
    _require(q, torch.int8, 2, "q", x.device)
    _require(s, torch.float32, 1, "s", x.device)
    if tuple(q.shape) != (M, K) or tuple(s.shape) != (M,):
        raise ValueError("output shapes do not match x")
    with torch.cuda.device(x.device):
        st = raw.tfq_quant_act_int8_per_token(x.data_ptr(), M, K, float(qmax), q.data_ptr(), s.data_ptr(),
                                              _stream_handle(stream))
    _check(st, "tfq_quant_act_int8_per_token")
    return q, s


def tfq_scaled_int8_linear(A_q, s_a, W_q, s_w, bias=None, out=None, stream=None):
    """A_q int8 [M, K], s_a fp32 [M], W_q int8 [N, K], s_w fp32 [N], bias bf16 [N] or None
    -> out bf16 [M, N]."""
    import torch
    _require(A_q, torch.int8, 2, "A_q")
    dev = A_q.device
    _require(W_q, torch.int8, 2, "W_q", dev)
    _require(s_a, torch.float32, 1, "s_a", dev)
    _require(s_w, torch.float32, 1, "s_w", dev)
    M, K = A_q.shape
    N, K2 = W_q.shape
    if K2 != K or s_a.shape[0] != M or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    if bias is not None:
        _require(bias, torch.bfloat16, 1, "bias", dev)
        if bias.shape[0] != N:
            raise ValueError("bias shape")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A_q.device)
    _require(out, torch.bfloat16, 2, "out", dev)
    if tuple(out.shape) != (M, N):
        raise ValueError("out shape")
    with torch.cuda.device(A_q.device):
        st = raw.tfq_scaled_int8_linear(A_q.data_ptr(), s_a.data_ptr(), W_q.data_ptr(), s_w.data_ptr(),
                                        None if bias is None else bias.data_ptr(), M, N, K, out.data_ptr(),
                                        _stream_handle(stream))
    _check(st, "tfq_scaled_int8_linear")
    return out


def w8a8_int8_linear(x, W_q, s_w, bias=None, qmax: float = 127.0, stream=None):
    """The INT8 Linear: per-token INT8 quantization of x, then the scaled INT8 GEMM."""
    A_q, s_a = tfq_quant_act_int8_per_token(x, qmax, stream=stream)
    return tfq_scaled_int8_linear(A_q, s_a, W_q, s_w, bias, stream=stream)


def tfq_mxfp8_scale_bytes(rows: int, K: int) -> int:
    """Bytes of the E8M0 scale buffer of a [rows, K] MXFP8 operand."""
    n = int(load_library().tfq_mxfp8_scale_bytes(int(rows), int(K)))
    if n < 0:
        raise ValueError("negative size")
    return n


def tfq_quant_mxfp8(x, q=None, sf=None, stream=None):
    """x bf16 [R, K] (K % 32 == 0) -> (q uint8 [R, K] E4M3FN codes,
    sf uint8 [tfq_mxfp8_scale_bytes(R, K)] E8M0 codes in the tensor-core layout)."""
    import torch
    _require(x, torch.bfloat16, 2, "x")
    R, K = x.shape
    if q is None:
        q = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((tfq_mxfp8_scale_bytes(R, K),), dtype=torch.uint8, device=x.device)
    _require(q, torch.uint8, 2, "q", x.device)
    _require(sf, torch.uint8, 1, "sf", x.device)
    if tuple(q.shape) != (R, K) or sf.numel() < tfq_mxfp8_scale_bytes(R, K):
        raise ValueError("output shapes do not match x")
    with torch.cuda.device(x.device):
        st = raw.tfq_quant_mxfp8(x.data_ptr(), R, K, q.data_ptr(), sf.data_ptr(), _stream_handle(stream))
    _check(st, "tfq_quant_mxfp8")
    return q, sf


def tfq_mxfp8_linear(A_q, sf_a, W_q, sf_w, bias=None, out=None, stream=None):
    """A_q uint8 [M, K], W_q uint8 [N, K] E4M3FN codes with their scale buffers
    from tfq_quant_mxfp8, bias bf16 [N] or None -> out bf16 [M, N]."""
    import torch
    _require(A_q, torch.uint8, 2, "A_q")
    dev = A_q.device
    _require(W_q, torch.uint8, 2, "W_q", dev)
    _require(sf_a, torch.uint8, 1, "sf_a", dev)
    _require(sf_w, torch.uint8, 1, "sf_w", dev)
    M, K = A_q.shape
    N, K2 = W_q.shape
    if K2 != K or sf_a.numel() < tfq_mxfp8_scale_bytes(M, K) or sf_w.numel() < tfq_mxfp8_scale_bytes(N, K):
        raise ValueError("shape mismatch")
    if bias is not None:
        _require(bias, torch.bfloat16, 1, "bias", dev)
        if bias.shape[0] != N:
            raise ValueError("bias shape")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A_q.device)
    _require(out, torch.bfloat16, 2, "out", dev)
    if tuple(out.shape) != (M, N):
        raise ValueError("out shape")
    with torch.cuda.device(A_q.device):
        st = raw.tfq_mxfp8_linear(A_q.data_ptr(), sf_a.data_ptr(), W_q.data_ptr(), sf_w.data_ptr(),
                                  None if bias is None else bias.data_ptr(), M, N, K, out.data_ptr(),
                                  _stream_handle(stream))
    _check(st, "tfq_mxfp8_linear")
    return out


def mxfp8_linear(x, W_q, sf_w, bias=None, stream=None):
    """The MXFP8 Linear: block quantization of x, then the block-scaled GEMM."""
    A_q, sf_a = tfq_quant_mxfp8(x, stream=stream)
    return tfq_mxfp8_linear(A_q, sf_a, W_q, sf_w, bias, stream=stream)


def tfq_device_error(stream=None) -> None:
    """Raises TfqError(TFQ_ETIMEOUT) if a bounded device wait ran out."""
    _check(raw.tfq_device_error(_stream_handle(stream)), "tfq_device_error")


def w8a8_linear(x, W_q, s_w, bias=None, qmax: float = 448.0, stream=None):
    """The whole Linear: per-token FP8 quantization of x, then the scaled GEMM."""
    A_q, s_a = tfq_quant_act_fp8_per_token(x, qmax, stream=stream)
    return tfq_scaled_fp8_linear(A_q, s_a, W_q, s_w, bias, stream=stream)


def pointer_array(ptrs):
    """A C array of void* (None for NULL entries) for the multi-Linear call."""
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def _linear_multi(name, code_dtype, A_q, s_a, W_qs, s_ws, biases, outs, stream):
    """The multi-Linear GEMM `name` on operands of `code_dtype`."""
    import torch
    n = len(W_qs)
    if not 1 <= n <= TFQ_MULTI_MAX_LINEARS or len(s_ws) != n or (biases is not None and len(biases) != n):
        raise ValueError(f"1 to {TFQ_MULTI_MAX_LINEARS} Linears with one weight, scale and bias entry each")
    _require(A_q, code_dtype, 2, "A_q")
    dev = A_q.device
    _require(s_a, torch.float32, 1, "s_a", dev)
    M, K = A_q.shape
    if s_a.shape[0] != M:
        raise ValueError("shape mismatch")
    biases = [None] * n if biases is None else list(biases)
    outs = [None] * n if outs is None else list(outs)
    Ns = []
    for i in range(n):
        _require(W_qs[i], code_dtype, 2, "W_q", dev)
        _require(s_ws[i], torch.float32, 1, "s_w", dev)
        N, K2 = W_qs[i].shape
        if K2 != K or s_ws[i].shape[0] != N:
            raise ValueError("shape mismatch")
        if biases[i] is not None:
            _require(biases[i], torch.bfloat16, 1, "bias", dev)
            if biases[i].shape[0] != N:
                raise ValueError("bias shape")
        if outs[i] is None:
            outs[i] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        _require(outs[i], torch.bfloat16, 2, "out", dev)
        if tuple(outs[i].shape) != (M, N):
            raise ValueError("out shape")
        Ns.append(N)
    with torch.cuda.device(dev):
        st = getattr(raw, name)(
            A_q.data_ptr(), s_a.data_ptr(), M, K, n, pointer_array([w.data_ptr() for w in W_qs]),
            pointer_array([s.data_ptr() for s in s_ws]),
            pointer_array([None if b is None else b.data_ptr() for b in biases]),
            (ctypes.c_int64 * n)(*Ns), pointer_array([o.data_ptr() for o in outs]), _stream_handle(stream))
    _check(st, name)
    return outs


def tfq_scaled_fp8_linear_multi(A_q, s_a, W_qs, s_ws, biases=None, outs=None, stream=None):
    """The Linears that share A_q, s_a: W_qs / s_ws / biases (lists, biases or
    any entry None) -> [out bf16 [M, N_i]], as one launch of the CTA-pair
    kernel from 512 rows up (same bits as separate tfq_scaled_fp8_linear calls)."""
    import torch
    return _linear_multi("tfq_scaled_fp8_linear_multi", torch.uint8, A_q, s_a, W_qs, s_ws, biases, outs, stream)


def tfq_scaled_int8_linear_multi(A_q, s_a, W_qs, s_ws, biases=None, outs=None, stream=None):
    """tfq_scaled_fp8_linear_multi with int8 operands (same bits as separate
    tfq_scaled_int8_linear calls)."""
    import torch
    return _linear_multi("tfq_scaled_int8_linear_multi", torch.int8, A_q, s_a, W_qs, s_ws, biases, outs, stream)


def tfq_quant_scaled_fp8_linear_workspace_bytes(M: int) -> int:
    """Bytes of the workspace tfq_quant_scaled_fp8_linear needs for M rows."""
    return int(load_library().tfq_quant_scaled_fp8_linear_workspace_bytes(int(M)))


def tfq_quant_scaled_fp8_linear(x, W_q, s_w, bias=None, qmax: float = 448.0, A_q=None, s_a=None, out=None,
                                workspace=None, stream=None):
    """x bf16 [M, K], W_q uint8 [N, K], s_w fp32 [N], bias bf16 [N] or None ->
    (out bf16 [M, N], A_q uint8 [M, K], s_a fp32 [M]): per-token FP8
    quantization of x and the scaled GEMM in one call (one kernel from 512
    rows up)."""
    import torch
    _require(x, torch.bfloat16, 2, "x")
    dev = x.device
    _require(W_q, torch.uint8, 2, "W_q", dev)
    _require(s_w, torch.float32, 1, "s_w", dev)
    M, K = x.shape
    N, K2 = W_q.shape
    if K2 != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    if bias is not None:
        _require(bias, torch.bfloat16, 1, "bias", dev)
        if bias.shape[0] != N:
            raise ValueError("bias shape")
    if A_q is None:
        A_q = torch.empty((M, K), dtype=torch.uint8, device=dev)
    if s_a is None:
        s_a = torch.empty((M,), dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    nws = tfq_quant_scaled_fp8_linear_workspace_bytes(M)
    if workspace is None:
        workspace = torch.empty((max(nws, 16),), dtype=torch.uint8, device=dev)
    _require(A_q, torch.uint8, 2, "A_q", dev)
    _require(s_a, torch.float32, 1, "s_a", dev)
    _require(out, torch.bfloat16, 2, "out", dev)
    _require(workspace, torch.uint8, 1, "workspace", dev)
    if tuple(A_q.shape) != (M, K) or tuple(s_a.shape) != (M,) or tuple(out.shape) != (M, N):
        raise ValueError("output shapes do not match x and W_q")
    if workspace.numel() < nws:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, {nws} needed")
    with torch.cuda.device(dev):
        st = raw.tfq_quant_scaled_fp8_linear(x.data_ptr(), M, K, float(qmax), W_q.data_ptr(), s_w.data_ptr(),
                                             None if bias is None else bias.data_ptr(), N, A_q.data_ptr(),
                                             s_a.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                                             _stream_handle(stream))
    _check(st, "tfq_quant_scaled_fp8_linear")
    return out, A_q, s_a
