// tfq_args.h -- host-side argument checks shared by the C-ABI entry points.
#pragma once

#include <cstdint>

#include "tfq.h"

namespace tfq {

// Checks of a scaled FP8 / INT8 GEMM call before any device work: sizes
// (K a positive multiple of 16, N a multiple of 8, each below 2^31), and,
// unless the output is empty, non-null 16-byte aligned operands (bias may be
// null).  Returns TFQ_OK or the status the call must return, with the
// message recorded for tfq_last_error_message().
tfq_status check_gemm_args(const void* A_q, const float* s_a, const void* W_q, const float* s_w,
                           const void* bias_bf16, int64_t M, int64_t N, int64_t K, const void* out_bf16);

}  // namespace tfq
