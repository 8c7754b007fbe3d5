"""B200-native (sm_100a) W8A8 scaled-FP8 Linear.

The computation lives in libtfq.so (include/tfq.h): a per-row absmax
quantizer (BF16 -> E4M3FN or INT8 with one fp32 scale per row) and a
tcgen05/TMEM/TMA scaled FP8 GEMM with a fused scale/bias/BF16 epilogue.
This package is its Python binding; torch supplies device memory and
streams.  Build the library with ``python -m int8_w8a8_quantized_b200.build``.
"""
from ._capi import (  # noqa: F401
    LIB_PATH,
    SIGNATURES,
    TFQ_DTYPE_FP8_E4M3,
    TFQ_DTYPE_INT8,
    TFQ_EINVAL,
    TFQ_ECUDA,
    TFQ_ETIMEOUT,
    TFQ_EUNSUPPORTED,
    TFQ_OK,
    TFQ_INT8_MAX_K,
    TFQ_QUANT_MAX_K,
    TfqError,
    last_error_message,
    load_library,
    mxfp8_linear,
    raw,
    status_string,
    tfq_device_error,
    tfq_mxfp8_linear,
    tfq_mxfp8_scale_bytes,
    tfq_quant_act_fp8_per_token,
    tfq_quant_act_int8_per_token,
    tfq_quant_mxfp8,
    tfq_quant_scaled_fp8_linear,
    tfq_quant_scaled_fp8_linear_workspace_bytes,
    tfq_quant_weight_per_channel,
    tfq_scaled_fp8_linear,
    tfq_scaled_fp8_linear_f16acc,
    tfq_scaled_fp8_linear_multi,
    tfq_scaled_fp8_linear_noalloc,
    tfq_scaled_int8_linear,
    tfq_scaled_int8_linear_multi,
    w8a8_int8_linear,
    w8a8_linear,
)

__all__ = [
    "tfq_quant_act_fp8_per_token",
    "tfq_quant_weight_per_channel",
    "tfq_scaled_fp8_linear",
    "tfq_quant_scaled_fp8_linear",
    "tfq_quant_scaled_fp8_linear_workspace_bytes",
    "tfq_scaled_fp8_linear_f16acc",
    "tfq_scaled_fp8_linear_multi",
    "tfq_scaled_fp8_linear_noalloc",
    "tfq_quant_act_int8_per_token",
    "tfq_scaled_int8_linear",
    "tfq_scaled_int8_linear_multi",
    "w8a8_int8_linear",
    "tfq_device_error",
    "w8a8_linear",
    "tfq_quant_mxfp8",
    "tfq_mxfp8_linear",
    "tfq_mxfp8_scale_bytes",
    "mxfp8_linear",
    "TfqError",
    "raw",
]
