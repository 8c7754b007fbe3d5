// tfq_capi.cu -- the extern "C" entry points of libtfq.so: argument
// validation, per-device state, TMA descriptor encoding, launches.
// See include/tfq.h for the contract of every function.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "tfq_args.h"
#include "tfq_internal.h"

namespace tfq {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
DeviceState g_states[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
thread_local char g_last_error[512] = "";

std::mutex g_encode_mutex;

}  // namespace

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tfq_status resolve_encode() {
    std::lock_guard<std::mutex> lock(g_encode_mutex);
    if (g_encode != nullptr) return TFQ_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                           cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return fail(TFQ_ECUDA, "cannot resolve cuTensorMapEncodeTiled: %s", cudaGetErrorString(e));
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return TFQ_OK;
}

tfq_status fail(tfq_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

DeviceState* current_device_state(tfq_status* st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *st = fail(TFQ_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *st = fail(TFQ_EUNSUPPORTED, "device ordinal %d out of range", dev);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState* ds = &g_states[dev];
    if (ds->device < 0) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) {
            *st = fail(TFQ_ECUDA, "cudaGetDeviceProperties: %s", cudaGetErrorString(e));
            return nullptr;
        }
        if (prop.major != 10 || prop.minor != 0) {
            *st = fail(TFQ_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, prop.major,
                       prop.minor);
            return nullptr;
        }
        tfq_status rs = resolve_encode();
        if (rs != TFQ_OK) {
            *st = rs;
            return nullptr;
        }
        // One allocation: the error word in the first 128-byte line, then
        // kRoundSlots round counters, one line each.
        constexpr int kRoundSlots = 64;
        uint32_t* err_word = nullptr;
        e = cudaMalloc(&err_word, 128 * (1 + kRoundSlots));
        if (e == cudaSuccess) e = cudaMemset(err_word, 0, 128 * (1 + kRoundSlots));
        if (e != cudaSuccess) {
            if (err_word != nullptr) cudaFree(err_word);
            *st = fail(TFQ_ECUDA, "allocating the device error word: %s", cudaGetErrorString(e));
            return nullptr;
        }
        ds->round_ctrs = err_word + 32;
        ds->round_slots = kRoundSlots;
        ds->sm_count = prop.multiProcessorCount;
        ds->cc_major = prop.major;
        ds->cc_minor = prop.minor;
        ds->smem_optin = prop.sharedMemPerBlockOptin;
        ds->err_word = err_word;
        ds->device = dev;
    }
    *st = TFQ_OK;
    return ds;
}

unsigned* take_round_counter(DeviceState* ds) {
    if (ds->round_ctrs == nullptr || ds->round_slots <= 0) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    const int slot = ds->next_round_slot;
    ds->next_round_slot = (slot + 1) % ds->round_slots;
    return ds->round_ctrs + 32 * slot;
}

tfq_status encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                                uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                                CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estride,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TFQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return TFQ_OK;
}

}  // namespace tfq

using namespace tfq;

namespace {

tfq_status check_quant_args(const void* x, int64_t M, int64_t K, const void* q, const float* s, float qmax,
                            float qmax_hi) {
    if (M < 0 || K < 0) return fail(TFQ_EINVAL, "negative size (M=%lld, K=%lld)", (long long)M, (long long)K);
    if (K % 16 != 0) return fail(TFQ_EINVAL, "K=%lld is not a multiple of 16", (long long)K);
    if (!std::isfinite(qmax) || qmax < 1.0f || qmax > qmax_hi)
        return fail(TFQ_EINVAL, "qmax=%g outside [1, %g]", (double)qmax, (double)qmax_hi);
    if (K > TFQ_QUANT_MAX_K) return fail(TFQ_EUNSUPPORTED, "K=%lld above %d", (long long)K, TFQ_QUANT_MAX_K);
    if (M >= (int64_t(1) << 31)) return fail(TFQ_EUNSUPPORTED, "M=%lld too large", (long long)M);
    if (M == 0) return TFQ_OK;
    if (s == nullptr || (K > 0 && (x == nullptr || q == nullptr)))
        return fail(TFQ_EINVAL, "null pointer");
    if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return fail(TFQ_EINVAL, "pointer not 16-byte aligned");
    return TFQ_OK;
}

}  // namespace

extern "C" {

tfq_status tfq_quant_act_fp8_per_token(const void* x_bf16, int64_t M, int64_t K, float qmax, void* q_e4m3,
                                       float* s, void* stream) {
    tfq_status st = check_quant_args(x_bf16, M, K, q_e4m3, s, qmax, 448.0f);
    if (st != TFQ_OK || M == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_quant_rows(x_bf16, M, K, qmax, false, q_e4m3, s, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_quant_weight_per_channel(const void* w_bf16, int64_t N, int64_t K, int dtype, float qmax, void* q,
                                        float* s, void* stream) {
    if (dtype != TFQ_DTYPE_FP8_E4M3 && dtype != TFQ_DTYPE_INT8) return fail(TFQ_EINVAL, "unknown dtype %d", dtype);
    const bool is_int8 = dtype == TFQ_DTYPE_INT8;
    tfq_status st = check_quant_args(w_bf16, N, K, q, s, qmax, is_int8 ? 127.0f : 448.0f);
    if (st != TFQ_OK || N == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_quant_rows(w_bf16, N, K, qmax, is_int8, q, s, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_quant_act_int8_per_token(const void* x_bf16, int64_t M, int64_t K, float qmax, void* q_int8,
                                        float* s, void* stream) {
    tfq_status st = check_quant_args(x_bf16, M, K, q_int8, s, qmax, 127.0f);
    if (st != TFQ_OK || M == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_quant_rows(x_bf16, M, K, qmax, true, q_int8, s, static_cast<cudaStream_t>(stream), ds);
}

}  // extern "C"

namespace tfq {

tfq_status check_gemm_args(const void* A_q, const float* s_a, const void* W_q, const float* s_w,
                           const void* bias_bf16, int64_t M, int64_t N, int64_t K, const void* out_bf16) {
    if (M < 0 || N < 0 || K < 0) return fail(TFQ_EINVAL, "negative size");
    if (K == 0 || K % 16 != 0) return fail(TFQ_EINVAL, "K=%lld must be a positive multiple of 16", (long long)K);
    if (N % 8 != 0) return fail(TFQ_EINVAL, "N=%lld is not a multiple of 8", (long long)N);
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return fail(TFQ_EUNSUPPORTED, "size too large");
    if (M == 0 || N == 0) return TFQ_OK;
    if (A_q == nullptr || s_a == nullptr || W_q == nullptr || s_w == nullptr || out_bf16 == nullptr)
        return fail(TFQ_EINVAL, "null pointer");
    if (!aligned16(A_q) || !aligned16(s_a) || !aligned16(W_q) || !aligned16(s_w) || !aligned16(out_bf16) ||
        (bias_bf16 != nullptr && !aligned16(bias_bf16)))
        return fail(TFQ_EINVAL, "pointer not 16-byte aligned");
    return TFQ_OK;
}

// The host checks of the multi-Linear GEMMs: n in [1, TFQ_MULTI_MAX_LINEARS],
// the arrays present and every Linear's arguments valid.
static tfq_status check_multi_args(const void* A_q, const float* s_a, int64_t M, int64_t K, int n,
                                   const void* const* W_q, const float* const* s_w, const void* const* bias_bf16,
                                   const int64_t* N, void* const* out_bf16) {
    if (n < 1 || n > TFQ_MULTI_MAX_LINEARS)
        return fail(TFQ_EINVAL, "n=%d outside [1, %d]", n, TFQ_MULTI_MAX_LINEARS);
    if (W_q == nullptr || s_w == nullptr || N == nullptr || out_bf16 == nullptr)
        return fail(TFQ_EINVAL, "null array");
    for (int i = 0; i < n; ++i) {
        const tfq_status st = check_gemm_args(A_q, s_a, W_q[i], s_w[i], bias_bf16 != nullptr ? bias_bf16[i] : nullptr,
                                              M, N[i], K, out_bf16[i]);
        if (st != TFQ_OK) return st;
    }
    return TFQ_OK;
}

using MultiLauncher = tfq_status (*)(const void*, const float*, int64_t, int64_t, int, const void* const*,
                                     const float* const*, const void* const*, const int64_t*, void* const*,
                                     cudaStream_t, DeviceState*);

static tfq_status launch_multi(MultiLauncher launcher, const void* A_q, const float* s_a, int64_t M, int64_t K,
                               int n, const void* const* W_q, const float* const* s_w, const void* const* bias_bf16,
                               const int64_t* N, void* const* out_bf16, void* stream) {
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launcher(A_q, s_a, M, K, n, W_q, s_w, bias_bf16, N, out_bf16, static_cast<cudaStream_t>(stream), ds);
}

}  // namespace tfq

extern "C" {

tfq_status tfq_scaled_int8_linear(const void* A_q, const float* s_a, const void* W_q, const float* s_w,
                                  const void* bias_bf16, int64_t M, int64_t N, int64_t K, void* out_bf16,
                                  void* stream) {
    tfq_status st = check_gemm_args(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16);
    if (st != TFQ_OK) return st;
    // |sum| <= 128^2 K must stay below 2^31 for the s32 accumulator to be exact
    if (K >= TFQ_INT8_MAX_K) return fail(TFQ_EUNSUPPORTED, "K=%lld: the INT8 sum may exceed s32 (K < %d)",
                                         (long long)K, TFQ_INT8_MAX_K);
    if (M == 0 || N == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_scaled_int8_gemm(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16,
                                   static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_scaled_fp8_linear_f16acc(const void* A_q, const float* s_a, const void* W_q, const float* s_w,
                                        const void* bias_bf16, int64_t M, int64_t N, int64_t K, void* out_bf16,
                                        void* stream) {
    tfq_status st = check_gemm_args(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16);
    if (st != TFQ_OK || M == 0 || N == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_scaled_fp8_gemm_f16acc(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16,
                                         static_cast<cudaStream_t>(stream), ds);
}

int64_t tfq_mxfp8_scale_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K < 0) return -1;
    return ((rows + 127) / 128) * ((K + 127) / 128) * 512;
}

tfq_status tfq_quant_mxfp8(const void* x_bf16, int64_t rows, int64_t K, void* q_e4m3, void* sf_e8m0,
                           void* stream) {
    if (rows < 0 || K < 0) return fail(TFQ_EINVAL, "negative size (rows=%lld, K=%lld)", (long long)rows, (long long)K);
    if (K % TFQ_MX_BLOCK != 0) return fail(TFQ_EINVAL, "K=%lld is not a multiple of %d", (long long)K, TFQ_MX_BLOCK);
    if (K > TFQ_QUANT_MAX_K) return fail(TFQ_EUNSUPPORTED, "K=%lld above %d", (long long)K, TFQ_QUANT_MAX_K);
    if (rows >= (int64_t(1) << 31)) return fail(TFQ_EUNSUPPORTED, "rows=%lld too large", (long long)rows);
    if (rows == 0 || K == 0) return TFQ_OK;
    if (x_bf16 == nullptr || q_e4m3 == nullptr || sf_e8m0 == nullptr) return fail(TFQ_EINVAL, "null pointer");
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sf_e8m0))
        return fail(TFQ_EINVAL, "pointer not 16-byte aligned");
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_quant_mxfp8(x_bf16, rows, K, q_e4m3, sf_e8m0, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_mxfp8_linear(const void* A_q, const void* sf_a, const void* W_q, const void* sf_w,
                            const void* bias_bf16, int64_t M, int64_t N, int64_t K, void* out_bf16, void* stream) {
    if (M < 0 || N < 0 || K < 0) return fail(TFQ_EINVAL, "negative size");
    if (K == 0 || K % TFQ_MX_BLOCK != 0)
        return fail(TFQ_EINVAL, "K=%lld must be a positive multiple of %d", (long long)K, TFQ_MX_BLOCK);
    if (N % 8 != 0) return fail(TFQ_EINVAL, "N=%lld is not a multiple of 8", (long long)N);
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return fail(TFQ_EUNSUPPORTED, "size too large");
    if (M == 0 || N == 0) return TFQ_OK;
    if (A_q == nullptr || sf_a == nullptr || W_q == nullptr || sf_w == nullptr || out_bf16 == nullptr)
        return fail(TFQ_EINVAL, "null pointer");
    if (!aligned16(A_q) || !aligned16(sf_a) || !aligned16(W_q) || !aligned16(sf_w) || !aligned16(out_bf16) ||
        (bias_bf16 != nullptr && !aligned16(bias_bf16)))
        return fail(TFQ_EINVAL, "pointer not 16-byte aligned");
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_mxfp8_gemm(A_q, static_cast<const uint8_t*>(sf_a), W_q, static_cast<const uint8_t*>(sf_w),
                             bias_bf16, M, N, K, out_bf16, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_scaled_fp8_linear(const void* A_q, const float* s_a, const void* W_q, const float* s_w,
                                 const void* bias_bf16, int64_t M, int64_t N, int64_t K, void* out_bf16,
                                 void* stream) {
    tfq_status st = check_gemm_args(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16);
    if (st != TFQ_OK || M == 0 || N == 0) return st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_scaled_fp8_gemm(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16,
                                  static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_scaled_fp8_linear_multi(const void* A_q, const float* s_a, int64_t M, int64_t K, int n,
                                       const void* const* W_q, const float* const* s_w, const void* const* bias_bf16,
                                       const int64_t* N, void* const* out_bf16, void* stream) {
    const tfq_status st = check_multi_args(A_q, s_a, M, K, n, W_q, s_w, bias_bf16, N, out_bf16);
    if (st != TFQ_OK || M == 0) return st;
    return launch_multi(launch_scaled_fp8_gemm_multi, A_q, s_a, M, K, n, W_q, s_w, bias_bf16, N, out_bf16, stream);
}

tfq_status tfq_scaled_int8_linear_multi(const void* A_q, const float* s_a, int64_t M, int64_t K, int n,
                                        const void* const* W_q, const float* const* s_w, const void* const* bias_bf16,
                                        const int64_t* N, void* const* out_bf16, void* stream) {
    const tfq_status st = check_multi_args(A_q, s_a, M, K, n, W_q, s_w, bias_bf16, N, out_bf16);
    if (st != TFQ_OK) return st;
    if (K >= TFQ_INT8_MAX_K) return fail(TFQ_EUNSUPPORTED, "K=%lld: the INT8 sum may exceed s32 (K < %d)",
                                         (long long)K, TFQ_INT8_MAX_K);
    if (M == 0) return st;
    return launch_multi(launch_scaled_int8_gemm_multi, A_q, s_a, M, K, n, W_q, s_w, bias_bf16, N, out_bf16, stream);
}

size_t tfq_quant_scaled_fp8_linear_workspace_bytes(int64_t M) {
    return M < 0 ? 0 : quant_gemm_workspace_bytes(M);
}

tfq_status tfq_quant_scaled_fp8_linear(const void* x_bf16, int64_t M, int64_t K, float qmax, const void* W_q,
                                       const float* s_w, const void* bias_bf16, int64_t N, void* A_q, float* s_a,
                                       void* out_bf16, void* workspace, void* stream) {
    tfq_status st = check_quant_args(x_bf16, M, K, A_q, s_a, qmax, 448.0f);
    if (st != TFQ_OK) return st;
    st = check_gemm_args(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16);
    if (st != TFQ_OK || M == 0) return st;
    if (workspace == nullptr || !aligned16(workspace))
        return fail(TFQ_EINVAL, "workspace null or not 16-byte aligned");
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_quant_scaled_fp8_gemm(x_bf16, M, K, qmax, !is_e4m3_value(qmax), W_q, s_w, bias_bf16, N, A_q, s_a,
                                        out_bf16, workspace, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_selftest_div_rn(const float* a, const float* b, int64_t n, float* ours, float* ieee,
                               void* stream) {
    if (n < 0) return fail(TFQ_EINVAL, "negative n");
    if (n == 0) return TFQ_OK;
    if (a == nullptr || b == nullptr || ours == nullptr || ieee == nullptr) return fail(TFQ_EINVAL, "null pointer");
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_div_selftest(a, b, n, ours, ieee, static_cast<cudaStream_t>(stream));
}

tfq_status tfq_selftest_wait_timeout(uint32_t limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 10000000u) return fail(TFQ_EINVAL, "limit_us=%u outside [1, 1e7]", limit_us);
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    return launch_wait_selftest(static_cast<uint64_t>(limit_us) * 1000u, static_cast<cudaStream_t>(stream), ds);
}

tfq_status tfq_device_error(void* stream) {
    tfq_status st;
    DeviceState* ds = current_device_state(&st);
    if (ds == nullptr) return st;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    uint32_t word = 0;
    e = cudaMemcpy(&word, ds->err_word, sizeof word, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && word != 0) e = cudaMemset(ds->err_word, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "reading the error word: %s", cudaGetErrorString(e));
    if (word != 0) return fail(TFQ_ETIMEOUT, "a bounded device wait ran out (error bits 0x%x)", word);
    return TFQ_OK;
}

const char* tfq_status_string(int status) {
    switch (status) {
        case TFQ_OK: return "TFQ_OK";
        case TFQ_EINVAL: return "TFQ_EINVAL";
        case TFQ_EUNSUPPORTED: return "TFQ_EUNSUPPORTED";
        case TFQ_ECUDA: return "TFQ_ECUDA";
        case TFQ_ETIMEOUT: return "TFQ_ETIMEOUT";
        default: return "unknown";
    }
}

const char* tfq_last_error_message(void) { return g_last_error; }

int tfq_version(void) { return 101; }

}  // extern "C"
