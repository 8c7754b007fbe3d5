// tfq_internal.h -- declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "tfq.h"

namespace tfq {

// Bits of the per-device error word (which role of which kernel gave up).
enum : uint32_t {
    kErrGemmProducer = 1u << 4,
    kErrGemmMma = 1u << 5,
    kErrGemmEpilogue = 1u << 6,
    kErrGemmDrain = 1u << 7,
    kErrSelfTest = 1u << 8,
    kErrQuantStage = 1u << 9,  // a staged-row quantizer gave up waiting for a row load
};

struct DeviceState {
    int device = -1;
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    size_t smem_optin = 0;          // max dynamic shared memory per block
    uint32_t* err_word = nullptr;   // device memory, one 32-bit word
    // Round counters of the GEMM's cluster pacing (one 128-byte line each:
    // the round count, then the count of clusters done); launches take slots
    // round-robin so that launches in flight at the same time on different
    // streams do not share one.  The last cluster of a launch to finish sets
    // both back to zero, so no memset precedes a launch.
    unsigned* round_ctrs = nullptr;
    int round_slots = 0;
    int next_round_slot = 0;
    // FP8, INT8, FP8/FP16 acc, MXFP8, MXFP8 pair, FP8 pair quantizing its activations
    bool gemm_attr_set[6] = {false, false, false, false, false, false};
    bool quant_attr_set = false;   // dynamic shared memory limit of the staged-row quantizers
};

#ifndef TFQ_PDL
#define TFQ_PDL 1  // launch the hot-path kernels with programmatic stream serialization
#endif

// Launches `kernel` on `stream`; with TFQ_PDL the launch may overlap the
// tail of the stream's previous kernel (the kernel calls pdl_wait() before
// touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = TFQ_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Per-device state of the current device, created on first use.  Returns
// nullptr and sets *st on failure.
DeviceState* current_device_state(tfq_status* st);

// Resolves cuTensorMapEncodeTiled through the runtime (once; thread safe).
tfq_status resolve_encode();

// True when p is 16-byte aligned.
bool aligned16(const void* p);

// Records a message for tfq_last_error_message() and returns `st`.
tfq_status fail(tfq_status st, const char* fmt, ...);

// cuTensorMapEncodeTiled, resolved through the runtime's driver entry point.
tfq_status encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                                uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                                CUtensorMapSwizzle swizzle);

// True when v is exactly representable in E4M3FN (at most 4 significant bits,
// within the normal range used for qmax): then an FP8 quantizer needs no
// clamp to +-qmax (x / s exceeds qmax by at most one rounding, which encodes
// like qmax).
bool is_e4m3_value(float v);

// Row quantizer: out_int8 == false -> E4M3FN codes, true -> INT8 codes.
tfq_status launch_quant_rows(const void* x, int64_t rows, int64_t K, float qmax, bool out_int8, void* q, float* s,
                             cudaStream_t stream, DeviceState* ds);

// MXFP8 quantizer (E4M3 codes, one E8M0 scale per 32 values).
tfq_status launch_quant_mxfp8(const void* x, int64_t rows, int64_t K, void* q, void* sf, cudaStream_t stream,
                              DeviceState* ds);

// Self-check: the quantizer's division next to the IEEE division.
tfq_status launch_div_selftest(const float* a, const float* b, int64_t n, float* ours, float* ieee,
                               cudaStream_t stream);

// Self-check of the bounded wait: a wait on a barrier that never completes.
tfq_status launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream, DeviceState* ds);

// Round-counter slot for the next GEMM launch on this device (thread safe).
unsigned* take_round_counter(DeviceState* ds);

// Scaled FP8 GEMM with the fused scale/bias/BF16 epilogue.
tfq_status launch_scaled_fp8_gemm(const void* A, const float* s_a, const void* W, const float* s_w,
                                  const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                  cudaStream_t stream, DeviceState* ds);

// Scaled FP8 GEMMs of n <= 4 Linears that share A_q and s_a: one launch of
// the CTA-pair kernel (their N tiles concatenated) from M = 512 rows up, one
// launch per Linear below.  bias may be null (no bias for any), and so may
// any bias[i]; Linears with N[i] == 0 are skipped.
tfq_status launch_scaled_fp8_gemm_multi(const void* A, const float* s_a, int64_t M, int64_t K, int n,
                                        const void* const* W, const float* const* s_w, const void* const* bias,
                                        const int64_t* N, void* const* out, cudaStream_t stream, DeviceState* ds);

// The same with int8 operands (S8 x S8 -> S32).
tfq_status launch_scaled_int8_gemm_multi(const void* A, const float* s_a, int64_t M, int64_t K, int n,
                                         const void* const* W, const float* const* s_w, const void* const* bias,
                                         const int64_t* N, void* const* out, cudaStream_t stream, DeviceState* ds);

// Bytes of the workspace of launch_quant_scaled_fp8_gemm for M rows.
size_t quant_gemm_workspace_bytes(int64_t M);

// Per-token FP8 quantization of x [M, K] into A (codes) and s_a (scales)
// and the scaled FP8 GEMM on them, in one kernel from M = 512 rows up (its
// quantizer warps overlap the quantization with the MMAs; `workspace`
// holds its row counters and is cleared on `stream` first), as the row
// quantizer followed by the GEMM below that.  clamp: qmax is not an E4M3
// value.
tfq_status launch_quant_scaled_fp8_gemm(const void* x, int64_t M, int64_t K, float qmax, bool clamp, const void* W,
                                        const float* s_w, const void* bias, int64_t N, void* A, float* s_a,
                                        void* out, void* workspace, cudaStream_t stream, DeviceState* ds);

// Scaled FP8 GEMM with a half-precision (FP16) accumulator.
tfq_status launch_scaled_fp8_gemm_f16acc(const void* A, const float* s_a, const void* W, const float* s_w,
                                         const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                         cudaStream_t stream, DeviceState* ds);

// MXFP8 GEMM (E4M3 x E4M3 with one E8M0 scale per 32 values of K on both
// operands, block-scaled on the tensor cores) with the bias/BF16 epilogue.
tfq_status launch_mxfp8_gemm(const void* A, const uint8_t* sf_a, const void* W, const uint8_t* sf_w, const void* bias,
                             int64_t M, int64_t N, int64_t K, void* out, cudaStream_t stream, DeviceState* ds);

// Scaled INT8 GEMM (S8 x S8 -> S32 on the tensor cores) with the same epilogue.
tfq_status launch_scaled_int8_gemm(const void* A, const float* s_a, const void* W, const float* s_w,
                                   const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                                   cudaStream_t stream, DeviceState* ds);

}  // namespace tfq
