// tfq_noalloc.cu -- tfq_scaled_fp8_linear_noalloc: the scaled FP8 GEMM for
// callers that cannot allocate device memory.
//
// Who needs it: the regular entry points allocate one small device buffer
// (the per-device word in which a kernel records that a bounded wait ran
// out, and the counters the GEMM's clusters use to keep pace) with
// cudaMalloc on their first call on a device.  Some callers cannot allow
// that: a host framework that owns every byte of device memory through its
// own pool and forbids libraries from calling cudaMalloc, or a serving
// process that reserved nearly all of HBM up front.  This entry point runs
// the same GEMM kernel, but the words the kernel writes live in a
// file-scope __device__ array, so no call allocates anything.
//
// What it guarantees: no cudaMalloc, cudaFree or other allocating call, on
// any call.  Every call still issues stream-ordered CUDA calls (a memset of
// the scratch words and the kernel launch), and the first call on a device
// also queries the device and looks up the array's address; so, like any
// call that launches work, it cannot be made from inside a host callback
// enqueued on a stream, and its first call on a device belongs outside
// stream capture.
//
// The array is part of the library image: every GPU that loads the library
// holds it until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "tfq_args.h"
#include "tfq_internal.h"

namespace tfq {
namespace {

static_assert(TFQ_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

// Shared by every call of tfq_scaled_fp8_linear_noalloc on a device.  In host
// code this name is only a stand-in for the symbol: the device address is
// obtained with cudaGetSymbolAddress at set-up.
static __device__ __align__(256) uint32_t g_noalloc_scratch[TFQ_NOALLOC_SCRATCH_BYTES / sizeof(uint32_t)];

// Scratch the GEMM needs per call: its error word (first 128-byte line) and
// the round counter of its cluster pacing (second line).
constexpr size_t kGemmScratchBytes = 128 + 2 * sizeof(unsigned);  // error word; pacing line: rounds, clusters done

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
DeviceState g_noalloc_states[kMaxDevices];

// Set-up of the current device, once: device checks and the device address
// of the scratch array.  Allocates nothing (cudaGetSymbolAddress may load
// this library's device code into the context on first use).
DeviceState* noalloc_state(tfq_status* st) {
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
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    DeviceState* ds = &g_noalloc_states[dev];
    if (ds->device < 0) {
        int major = 0, minor = 0, sms = 0, smem_optin = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) {
            *st = fail(TFQ_ECUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
            return nullptr;
        }
        if (major != 10 || minor != 0) {
            *st = fail(TFQ_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
            return nullptr;
        }
        uint32_t* ptr = nullptr;
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            *st = fail(TFQ_ECUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
            return nullptr;
        }
        const tfq_status rs = resolve_encode();
        if (rs != TFQ_OK) {
            *st = rs;
            return nullptr;
        }
        ds->sm_count = sms;
        ds->cc_major = major;
        ds->cc_minor = minor;
        ds->smem_optin = static_cast<size_t>(smem_optin);
        ds->err_word = ptr;
        ds->round_ctrs = ptr + 32;  // one slot: calls overlapping on the GPU share it
        ds->round_slots = 1;
        ds->device = dev;
    }
    *st = TFQ_OK;
    return ds;
}

}  // namespace
}  // namespace tfq

using namespace tfq;

extern "C" tfq_status tfq_scaled_fp8_linear_noalloc(const void* A_q, const float* s_a, const void* W_q,
                                                    const float* s_w, const void* bias_bf16, int64_t M, int64_t N,
                                                    int64_t K, void* out_bf16, void* stream) {
    tfq_status st = check_gemm_args(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16);
    if (st != TFQ_OK) return st;
    if (kGemmScratchBytes > TFQ_NOALLOC_SCRATCH_BYTES)
        return fail(TFQ_EUNSUPPORTED, "call needs %zu bytes of scratch, the static array holds %d",
                    kGemmScratchBytes, TFQ_NOALLOC_SCRATCH_BYTES);
    if (M == 0 || N == 0) return TFQ_OK;
    DeviceState* ds = noalloc_state(&st);
    if (ds == nullptr) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the error word and both
    // pacing words must start at zero.  (The kernel's last cluster leaves the
    // pacing words at zero, but a call that overlapped another one on the
    // GPU, or whose waits gave up, may not have.)
    const cudaError_t e = cudaMemsetAsync(ds->err_word, 0, kGemmScratchBytes, s);
    if (e != cudaSuccess) return fail(TFQ_ECUDA, "clearing the scratch word: %s", cudaGetErrorString(e));
    return launch_scaled_fp8_gemm(A_q, s_a, W_q, s_w, bias_bf16, M, N, K, out_bf16, s, ds);
}
