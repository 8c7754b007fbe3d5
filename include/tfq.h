/*
 * tfq.h -- C ABI of libtfq.so, a B200 (sm_100a) W8A8 scaled-FP8 Linear.
 *
 * The Linear the source pages describe is two steps:
 *   1. per-token dynamic absmax quantization of BF16 activations to E4M3FN,
 *        s[m] = max_k |x[m,k]| / qmax,  q[m,k] = cast_E4M3FN(clamp(x[m,k] / s[m]))
 *      (TeleFuser "Quantization" page, section "Scaled FP8 checkpoints: W8A8";
 *       qmax 14 and 7 from the LightX2V "模型量化技术" page, section
 *       "MiniMax-H3 FP8 FP16 累加");
 *   2. a scaled GEMM against per-output-channel FP8 weights with BF16 output,
 *        y[m,n] = s_a[m] * s_w[n] * sum_k q_a[m,k] * q_w[n,k]  (+ bias[n])
 *      (same TeleFuser page, sections "Scaled FP8 checkpoints" and
 *       "tf-kernel FP8: online W8A8").
 * The per-output-channel weight converter (FP8, or INT8 with
 *   s = max|x| / 127, q = clamp(round(x / s), -128, 127),
 * TeleFuser "Quantization" page, sections "Core ideas" and "Offline
 * conversion") ships in the same library.
 *
 * Conventions shared by every entry point:
 *  - Every data pointer is a DEVICE pointer owned by the caller; the library
 *    never frees or keeps it.  Matrices are dense and row-major; a row is
 *    K contiguous elements.  E4M3FN codes and INT8 codes are bytes with the
 *    same bit patterns as torch.float8_e4m3fn / torch.int8.  Scales are fp32.
 *  - Every data pointer must be 16-byte aligned, and K must be a multiple
 *    of 16 (rows are then 16-byte aligned too).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream of the current device).  Work is enqueued asynchronously on it
 *    on the CURRENT device; the call returns once the launch is enqueued.
 *    Kernels are launched with programmatic stream serialization: a kernel
 *    may be scheduled and set itself up while the stream's previous kernel
 *    finishes, but reads and writes memory only after that kernel has
 *    completed, so stream order is kept.
 *  - Return value: TFQ_OK, or an error detected before any launch
 *    (TFQ_EINVAL for bad arguments, TFQ_EUNSUPPORTED for a device that is
 *    not sm_100 or a size beyond a stated limit), or TFQ_ECUDA when the CUDA
 *    runtime reports a launch error.  Nothing is launched when an argument
 *    check fails.
 *  - Device-side failures: every wait inside the kernels is bounded; a wait
 *    that runs out sets a per-device error word and the kernel returns.
 *    tfq_device_error() reports and clears it (TFQ_ETIMEOUT).
 *  - Rounding is fixed so that results are reproducible bit for bit:
 *    the scale is the fp32 IEEE quotient max(amax, 1e-12) / qmax, the
 *    element quotient x / s is an fp32 IEEE division, the FP8 cast rounds
 *    to nearest even and saturates, the INT8 rounding is half-to-even.
 *  - Thread safety: calls may come from several host threads; the library
 *    keeps per-device state (launch attributes, the error word, the GEMM's
 *    ring of cluster-pacing counters) behind a mutex.  TMA descriptors are
 *    encoded on the host for every call and passed as kernel parameters.
 *    The pacing ring has 64 slots taken in turn: more GEMMs than that in
 *    flight at once on one device (on many streams) can share a slot, which
 *    only loosens or delays the pacing (each wait gives up after 200 us);
 *    results never depend on it.
 *  - Non-finite inputs (inf, NaN) are outside the contract: the codes and
 *    scales of a row holding one are unspecified.
 *  - An output buffer must not overlap any input or any other output of the
 *    same call; the results are unspecified otherwise.
 */
#ifndef TFQ_H_
#define TFQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TFQ_API __attribute__((visibility("default")))
#else
#define TFQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tfq_status {
    TFQ_OK = 0,
    TFQ_EINVAL = 1,        /* null/misaligned pointer, bad size or qmax      */
    TFQ_EUNSUPPORTED = 2,  /* not an sm_100 device, or a size beyond a limit  */
    TFQ_ECUDA = 3,         /* the CUDA runtime reported an error              */
    TFQ_ETIMEOUT = 4       /* a bounded device-side wait ran out             */
} tfq_status;

/* Output element type of the per-row weight quantizer. */
enum { TFQ_DTYPE_FP8_E4M3 = 0, TFQ_DTYPE_INT8 = 1 };

/* Largest K (row length) the row quantizers accept (keeps the kernels' index
 * arithmetic in 32 bits).  Larger K returns TFQ_EUNSUPPORTED. */
#define TFQ_QUANT_MAX_K (1 << 24)

/*
 * Per-token FP8 activation quantization (step 1 above).
 *   x_bf16 : [M, K] bf16, read only.
 *   qmax   : fp32, 1 <= qmax <= 448 (the pages use 448, 14 and 7).
 *   q_e4m3 : [M, K] bytes, written: E4M3FN codes of clamp(x/s, -qmax, qmax).
 *   s      : [M] fp32, written: s[m] = fl32(max(amax_m, 1e-12f) / qmax).
 * M == 0 is a no-op.  K == 0 writes s only (amax of an empty row is 0).
 * Errors: TFQ_EINVAL (null or misaligned pointer with M > 0, M or K < 0,
 * K % 16 != 0, qmax outside [1, 448] or not finite), TFQ_EUNSUPPORTED
 * (K > TFQ_QUANT_MAX_K, M >= 2^31, not sm_100).
 */
TFQ_API tfq_status tfq_quant_act_fp8_per_token(const void *x_bf16, int64_t M, int64_t K, float qmax,
                                       void *q_e4m3, float *s, void *stream);

/*
 * Per-output-channel weight quantization: the same row quantizer applied to
 * the rows (output channels) of an nn.Linear weight [N, K].
 *   dtype == TFQ_DTYPE_FP8_E4M3 : as tfq_quant_act_fp8_per_token, qmax in [1, 448];
 *   dtype == TFQ_DTYPE_INT8     : s[n] = fl32(max(amax_n, 1e-12f) / qmax),
 *                                 q = clamp(round_half_even(fl32(w / s)), -128, 127),
 *                                 qmax in [1, 127] (the pages use 127).
 *   q : [N, K] bytes (E4M3FN codes or int8), s : [N] fp32.
 * Errors as for tfq_quant_act_fp8_per_token; an unknown dtype is TFQ_EINVAL.
 */
TFQ_API tfq_status tfq_quant_weight_per_channel(const void *w_bf16, int64_t N, int64_t K, int dtype,
                                        float qmax, void *q, float *s, void *stream);

/*
 * Scaled FP8 Linear (step 2 above), "TN": both operands K-contiguous.
 *   A_q  : [M, K] E4M3FN codes (per-token quantized activations).
 *   s_a  : [M] fp32 per-token scales.
 *   W_q  : [N, K] E4M3FN codes (per-output-channel quantized weight).
 *   s_w  : [N] fp32 per-channel scales.
 *   bias_bf16 : [N] bf16, or NULL for no bias.
 *   out_bf16  : [M, N] bf16, written:
 *       out[m,n] = bf16_rn(fp32(sum_k A_q[m,k] W_q[n,k]) * s_a[m] * s_w[n] + bias[n]).
 * The products are accumulated in fp32 on the tensor cores; the result is
 * within |y - y_exact| <= 2^-7 |y_exact| + 1e-3 rms(y_exact) of the exact
 * value (the tests check this bound).
 * M == 0 or N == 0 is a no-op.
 * Errors: TFQ_EINVAL (null/misaligned pointer, K <= 0, K % 16 != 0,
 * N % 8 != 0, negative sizes), TFQ_EUNSUPPORTED (M, N or K >= 2^31,
 * not sm_100).
 */
TFQ_API tfq_status tfq_scaled_fp8_linear(const void *A_q, const float *s_a, const void *W_q,
                                 const float *s_w, const void *bias_bf16, int64_t M, int64_t N,
                                 int64_t K, void *out_bf16, void *stream);

/* Most Linears tfq_scaled_fp8_linear_multi and tfq_scaled_int8_linear_multi take in one call. */
#define TFQ_MULTI_MAX_LINEARS 4

/*
 * Scaled FP8 Linears that share their input: out[i] = the result of
 * tfq_scaled_fp8_linear(A_q, s_a, W_q[i], s_w[i], bias_bf16[i], M, N[i], K,
 * out[i]) for i < n, 1 <= n <= TFQ_MULTI_MAX_LINEARS -- such as the Q, K and
 * V projections of a DiT block, which read one normed input (the per-token
 * quantized activations A_q, s_a).  The arrays are host arrays of n entries;
 * bias_bf16 may be NULL (no bias for any Linear), and so may any
 * bias_bf16[i].  From M = 512 rows up the n GEMMs run as one launch of the
 * CTA-pair kernel, their N tiles concatenated, which saves the fixed costs
 * of n - 1 launches (ramp-up, drain, a partial last round); the results are
 * the same, bit for bit, as those of the n separate calls.  Each N[i] follows
 * the rules of tfq_scaled_fp8_linear (N[i] == 0 skips that Linear).
 * Errors: those of tfq_scaled_fp8_linear for any Linear, TFQ_EINVAL for n out
 * of range or a null array.
 */
TFQ_API tfq_status tfq_scaled_fp8_linear_multi(const void *A_q, const float *s_a, int64_t M, int64_t K, int n,
                                               const void *const *W_q, const float *const *s_w,
                                               const void *const *bias_bf16, const int64_t *N,
                                               void *const *out_bf16, void *stream);

/*
 * Per-token FP8 quantization and the scaled FP8 Linear in one call: the
 * LinearFP8 forward of the TeleFuser "Quantization" page (section "Scaled
 * FP8 checkpoints: W8A8": quantize each input row dynamically, then run the
 * scaled GEMM), with the per-token activation / per-output-channel weight
 * scheme of its section "tf-kernel FP8: online W8A8".
 *   x_bf16 : [M, K] bf16 activations, read only; qmax as in
 *            tfq_quant_act_fp8_per_token.
 *   W_q, s_w, bias_bf16, N : as in tfq_scaled_fp8_linear.
 *   A_q : [M, K] bytes, written: the E4M3FN codes tfq_quant_act_fp8_per_token
 *         writes (bit for bit); s_a : [M] fp32, written: its scales.
 *   out_bf16 : [M, N] bf16, written: as tfq_scaled_fp8_linear(A_q, s_a, ...).
 *   workspace : device memory of
 *         tfq_quant_scaled_fp8_linear_workspace_bytes(M) bytes, owned by the
 *         caller, 16-byte aligned; cleared by the call on `stream` (so calls
 *         that overlap on the GPU need workspaces of their own).
 * From M = 512 rows up one kernel does both: besides the GEMM's roles every
 * CTA runs quantizer warps that quantize rows in increasing order ahead of
 * the tiles that read them (each 128-row share is published through a
 * counter in the workspace, and a CTA waits, bounded, for the shares it
 * loads), so the HBM-bound quantization overlaps the tensor-bound GEMM.
 * Below 512 rows it runs the row quantizer, then the GEMM.  A_q and s_a stay
 * valid after the call (the other Linears of a shared input, such as K and V
 * beside Q, can take them to tfq_scaled_fp8_linear).
 * Measured on B200 the one-kernel form is not faster than the two calls
 * tfq_quant_act_fp8_per_token + tfq_scaled_fp8_linear (the GEMM slows down by
 * about the quantizer's time); those remain the recommended path, and this
 * entry point is the measured alternative (same results, bit for bit).
 * M == 0 is a no-op; N == 0 quantizes only.
 * Errors: those of tfq_quant_act_fp8_per_token and tfq_scaled_fp8_linear,
 * TFQ_EINVAL for a null or misaligned workspace; a bounded wait that runs
 * out is reported by tfq_device_error() (TFQ_ETIMEOUT).
 */
TFQ_API size_t tfq_quant_scaled_fp8_linear_workspace_bytes(int64_t M);
TFQ_API tfq_status tfq_quant_scaled_fp8_linear(const void *x_bf16, int64_t M, int64_t K, float qmax,
                                               const void *W_q, const float *s_w, const void *bias_bf16,
                                               int64_t N, void *A_q, float *s_a, void *out_bf16,
                                               void *workspace, void *stream);

/*
 * INT8 W8A8 (the int8 modes of the LightX2V "模型量化技术" page, quantization-
 * mode table: INT8 per-channel symmetric weights, dynamic per-token symmetric
 * INT8 activations), with the integer formula of the TeleFuser
 * "Quantization" page, section "Core ideas".
 *
 * tfq_quant_act_int8_per_token: x bf16 [M, K] -> q int8 [M, K],
 *   s[m] = fl32(max(amax_m, 1e-12f) / qmax),
 *   q = clamp(round_half_even(fl32(x / s)), -128, 127); qmax in [1, 127]
 *   (the pages use 127).  Same preconditions and errors as
 *   tfq_quant_act_fp8_per_token.
 */
TFQ_API tfq_status tfq_quant_act_int8_per_token(const void *x_bf16, int64_t M, int64_t K, float qmax,
                                                void *q_int8, float *s, void *stream);

/*
 * tfq_scaled_int8_linear: as tfq_scaled_fp8_linear with int8 operands:
 *   A_q int8 [M, K], W_q int8 [N, K] (both K-contiguous), s_a [M], s_w [N]
 *   fp32, bias bf16 [N] or NULL, out bf16 [M, N]:
 *   out[m,n] = bf16_rn(fp32(sum_k A_q[m,k] W_q[n,k]) * s_a[m] * s_w[n] + bias[n]),
 * the integer sum exact in s32 on the tensor cores (|sum| <= 128^2 K < 2^31
 * for K < TFQ_INT8_MAX_K = 131072), converted to fp32 (round to nearest) in
 * the epilogue.  Same preconditions, tolerance and errors as
 * tfq_scaled_fp8_linear, and K >= TFQ_INT8_MAX_K returns TFQ_EUNSUPPORTED.
 */
#define TFQ_INT8_MAX_K 131072
TFQ_API tfq_status tfq_scaled_int8_linear(const void *A_q, const float *s_a, const void *W_q,
                                          const float *s_w, const void *bias_bf16, int64_t M, int64_t N,
                                          int64_t K, void *out_bf16, void *stream);

/*
 * tfq_scaled_int8_linear_multi: tfq_scaled_fp8_linear_multi with int8
 * operands -- out[i] = the result of tfq_scaled_int8_linear(A_q, s_a,
 * W_q[i], s_w[i], bias_bf16[i], M, N[i], K, out[i]) for i < n, the same bits,
 * from M = 512 rows up as one launch of the INT8 CTA-pair kernel.  Arrays,
 * preconditions and errors as in tfq_scaled_fp8_linear_multi, and K >=
 * TFQ_INT8_MAX_K returns TFQ_EUNSUPPORTED.
 */
TFQ_API tfq_status tfq_scaled_int8_linear_multi(const void *A_q, const float *s_a, int64_t M, int64_t K, int n,
                                                const void *const *W_q, const float *const *s_w,
                                                const void *const *bias_bf16, const int64_t *N,
                                                void *const *out_bf16, void *stream);

/*
 * tfq_scaled_fp8_linear_f16acc: tfq_scaled_fp8_linear with the products
 * accumulated in FP16 on the tensor cores instead of FP32 (the fp8-f16-accum
 * mode of the LightX2V "模型量化技术" page, quantization-mode table and
 * section "MiniMax-H3 FP8 FP16 累加"); the accumulator is widened to fp32 for
 * the epilogue.  A partial sum beyond +-65504 becomes +-inf and the output
 * element is then non-finite: that page lowers the activation qmax (14 or 7)
 * to keep the accumulator in range.  The result carries FP16 rounding of the
 * partial sums, so it is not held to tfq_scaled_fp8_linear's tolerance.
 * Same arguments, preconditions and errors as tfq_scaled_fp8_linear.
 */
TFQ_API tfq_status tfq_scaled_fp8_linear_f16acc(const void *A_q, const float *s_a, const void *W_q,
                                                const float *s_w, const void *bias_bf16, int64_t M, int64_t N,
                                                int64_t K, void *out_bf16, void *stream);

/*
 * MXFP8: E4M3FN codes with one E8M0 scale (a power of two 2^(c - 127), code
 * c in 0..254) per block of 32 consecutive elements of a row -- the format
 * the TeleFuser "Quantization" page names in section "Offline conversion"
 * (32-value blocks, E8M0 scales).  The page gives no conversion rule; the one
 * implemented is that of the OCP Microscaling (MX) v1.0 specification:
 *   E = floor(log2(max |x| over the block)) - 8, clamped to [-127, 127]
 *       (8 = exponent of 448, the largest E4M3 normal), code E + 127;
 *   q = E4M3FN_rn(clamp(x / 2^E, -448, 448))   (x / 2^E is exact);
 *   a block of zeros gets code 0.
 *
 * Scale-factor layout (the one the sm_100 block-scaled tensor-core MMA reads
 * from shared memory), for an operand of `rows` rows and K columns: with
 * RA = ceil(rows / 128) and KA = ceil(K / 128), the buffer holds RA * KA
 * atoms of 512 bytes; the atom of rows 128 ra.. and K blocks 4 ka.. is atom
 * number ka * RA + ra, and inside it the code of row r, K block b (b = k / 32)
 * is at byte 16 (r % 32) + 4 ((r % 128) / 32) + (b % 4).  Entries of rows >=
 * rows or blocks >= K / 32 are padding, written as 127 (scale 1) by
 * tfq_quant_mxfp8.  tfq_mxfp8_scale_bytes gives the buffer size.
 */
#define TFQ_MX_BLOCK 32
TFQ_API int64_t tfq_mxfp8_scale_bytes(int64_t rows, int64_t K);

/*
 * tfq_quant_mxfp8: x bf16 [rows, K] (row-major) -> q [rows, K] E4M3FN codes
 * and sf (tfq_mxfp8_scale_bytes(rows, K) bytes, layout above).  Activations
 * (rows = tokens) and weights (rows = output channels) alike.
 * Preconditions: K % 32 == 0, K <= TFQ_QUANT_MAX_K; 16-byte aligned pointers.
 * rows == 0 is a no-op.  Errors as tfq_quant_act_fp8_per_token.
 */
TFQ_API tfq_status tfq_quant_mxfp8(const void *x_bf16, int64_t rows, int64_t K, void *q_e4m3, void *sf_e8m0,
                                   void *stream);

/*
 * tfq_mxfp8_linear: the block-scaled GEMM, "TN":
 *   out[m,n] = bf16_rn(sum_b 2^(sfa[m,b]-127) 2^(sfw[n,b]-127)
 *                        sum_{k in block b} A_q[m,k] W_q[n,k] + bias[n])
 * with A_q [M, K], W_q [N, K] E4M3FN codes and sf_a, sf_w their scale
 * buffers from tfq_quant_mxfp8 (or any buffer in that layout with finite
 * codes <= 254).  The tensor cores apply both scales per 32-element block and
 * accumulate in fp32; tolerance as tfq_scaled_fp8_linear.
 * Preconditions: K % 32 == 0, N % 8 == 0, 16-byte aligned pointers.
 * Errors as tfq_scaled_fp8_linear.
 */
TFQ_API tfq_status tfq_mxfp8_linear(const void *A_q, const void *sf_a, const void *W_q, const void *sf_w,
                                    const void *bias_bf16, int64_t M, int64_t N, int64_t K, void *out_bf16,
                                    void *stream);

/*
 * Bytes of the static device array used by tfq_scaled_fp8_linear_noalloc.
 * Every GPU that loads the library holds this array until the process exits.
 */
#define TFQ_NOALLOC_SCRATCH_BYTES 256

/*
 * tfq_scaled_fp8_linear without any device allocation.  (An addition of this
 * library for callers that cannot allocate; the pages have no counterpart.)
 *
 * Same arguments, preconditions, result and errors as tfq_scaled_fp8_linear.
 * The regular entry points cudaMalloc one small device buffer per device on
 * their first call (the word where a kernel records a bounded wait that ran
 * out, and the counters the GEMM's clusters keep pace with).  Callers that
 * must not allocate device memory -- a framework that owns all device memory
 * through its own pool, a process that has reserved nearly all of HBM --
 * call this one instead: those words live in a file-scope __device__ array
 * of TFQ_NOALLOC_SCRATCH_BYTES bytes, and no call allocates (no cudaMalloc,
 * cudaFree or allocating library routine).
 *  - The caller still owns and passes every input and output.
 *  - A call needs 136 bytes of the array whatever M, N and K (the error
 *    word and, one 128-byte line further, two counters the kernel's clusters
 *    use to keep pace); a call needing more than the array holds is rejected
 *    with TFQ_EUNSUPPORTED.
 *  - The first call on a device does a one-time set-up with that device
 *    current (device checks, cudaGetSymbolAddress of the array, which may
 *    load the library's device code into the context); make that first call
 *    before any stream capture.
 *  - Every call issues stream-ordered CUDA calls (a memset and a kernel
 *    launch), so it cannot be made where CUDA calls are not allowed, such as
 *    inside a host callback enqueued on a stream.
 *  - Every call on a device shares the array, which keeps the last call's
 *    contents; each call clears those 136 bytes on `stream` before its
 *    kernel.  Calls that overlap on the GPU (on different streams) race on
 *    them (the counters only pace the clusters; results stay correct).
 *  - A bounded wait that runs out is recorded in the array's word only:
 *    this entry point does not read it back (that would need a host
 *    synchronization), and tfq_device_error() does not see it.
 */
TFQ_API tfq_status tfq_scaled_fp8_linear_noalloc(const void *A_q, const float *s_a, const void *W_q,
                                                 const float *s_w, const void *bias_bf16, int64_t M,
                                                 int64_t N, int64_t K, void *out_bf16, void *stream);

/*
 * Self-check of the division the quantizers use (a branch-free correctly
 * rounded fp32 division from a two-term reciprocal of the row scale and one
 * Markstein correction; the pages fix x / s, see the conventions above).
 * For i < n writes
 *   ours[i] = the quantizers' quotient a[i] / b[i],
 *   ieee[i] = the CUDA IEEE round-to-nearest quotient __fdiv_rn(a[i], b[i]);
 * the two agree bit for bit when |a / b| >= 2^-58 and 2^-49 <= b <= 2^64
 * (every row scale the quantizers use this division for); for smaller
 * |a / b| both quotients are below 2^-53 in magnitude with the sign of a,
 * so they give the same E4M3 and INT8 codes.  All pointers are device
 * pointers of n floats, 4-byte aligned.  Errors: TFQ_EINVAL (n < 0, null
 * pointer with n > 0).
 */
TFQ_API tfq_status tfq_selftest_div_rn(const float *a, const float *b, int64_t n, float *ours, float *ieee,
                                       void *stream);

/*
 * Self-check of the failure path: launches one tiny kernel whose only wait
 * is on a barrier that never completes, with the bounded-wait helper every
 * kernel here uses but a limit of limit_us microseconds (1 <= limit_us <=
 * 10^7) instead of the kernels' seconds.  The wait runs out, the kernel
 * records it in the device error word and returns; the next
 * tfq_device_error() then reports TFQ_ETIMEOUT and clears the word, and
 * the CUDA context stays usable.  Errors: TFQ_EINVAL (limit out of range).
 */
TFQ_API tfq_status tfq_selftest_wait_timeout(uint32_t limit_us, void *stream);

/*
 * Synchronizes `stream`, then reads and clears the current device's error
 * word.  Returns TFQ_ETIMEOUT if a bounded wait inside a kernel ran out
 * since the last call (the outputs of that launch are then incomplete),
 * TFQ_ECUDA if the synchronization itself failed, TFQ_OK otherwise.
 */
TFQ_API tfq_status tfq_device_error(void *stream);

/* Static string naming a status ("TFQ_OK", ...); "unknown" otherwise. */
TFQ_API const char *tfq_status_string(int status);

/* Thread-local text of the last error this thread's calls returned. */
TFQ_API const char *tfq_last_error_message(void);

/* ABI version: 100 * major + minor.  1.1 (101) added tfq_quant_scaled_fp8_linear,
 * tfq_scaled_fp8_linear_multi and tfq_scaled_int8_linear_multi to 1.0. */
TFQ_API int tfq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TFQ_H_ */
