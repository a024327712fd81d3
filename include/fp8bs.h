/*
 * fp8bs: FP8 block-scaled linear-layer kernels for NVIDIA B200 (sm_100a).
 *
 * C ABI of libfp8bs.so.  Every entry point takes plain pointers and sizes and
 * a CUDA stream passed as void* (a cudaStream_t; NULL is the legacy default
 * stream).  Unless stated otherwise, tensor pointers are DEVICE pointers owned
 * by the caller, row-major and contiguous, and must be 16-byte aligned.
 *
 * Calls are asynchronous.  Argument errors are detected on the host and are
 * returned before anything is launched.  A failed CUDA launch returns
 * FP8BS_ERR_CUDA.  Kernel-side failures (a bounded device wait that gave up)
 * are recorded in a per-device error word that fp8bs_get_device_error()
 * reads and clears.  fp8bs_last_error_message() describes the last non-OK
 * status returned on the calling host thread.
 *
 * The library allocates no device memory per call.  Kernels that need
 * scratch space take it from a caller-provided workspace whose size the
 * matching *_workspace_size() function returns.
 *
 * Per-device set-up (kernel attributes, the tensor-map encoder, the static
 * scratch array's address) is done on the first call that needs it on each
 * device and kept for the life of the process.  After cudaDeviceReset() of a
 * device, no entry point of this library may be called on that device again
 * in the same process: the kept set-up would refer to the destroyed context.
 *
 * Sources of the operations (page title, then section):
 *  [ACT] "Understanding Dynamic and Static Activation Quantization Schemes in
 *        DeepSeek-V3", "How Dynamic Activation Quantization Works";
 *        "DeepSeek-V3 quantization_config Parameters Explained: e4m3,
 *        weight_block_size, and activation_scheme", "The activation_scheme
 *        Parameter" and "The fmt Parameter".
 *  [DEQ] "How weight_dequant Handles Per-Block Scaling in DeepSeek-V3 FP8
 *        GEMM", "Grid Mapping and Scale Lookup", "Dequantization
 *        Computation", "Python Wrapper and Launch Configuration".
 *  [GEMM] same page, "Relationship to FP8 GEMM Operations" (fp8_gemm(a, a_s,
 *        b, b_s), scaling fused into the matrix product); "DeepSeek-V3: How
 *        Selective FP8 Stays Stable", "Learning outcomes" (1x128 activation
 *        tiles, 128x128 weight blocks, FP32 promotion of partial sums).
 *  [TRAIN] "DeepSeek-V3: How Selective FP8 Stays Stable", "Lower precision is
 *        a constrained budget" (forward, activation-gradient and
 *        weight-gradient GEMMs in FP8, outputs BF16 or FP32, weight gradients
 *        FP32).
 *  [STATIC] "Understanding Dynamic and Static Activation Quantization Schemes
 *        in DeepSeek-V3", "How Static Activation Quantization Differs"
 *        (precomputed scales; static_dequant multiplies the codes by them).
 */
#ifndef FP8BS_H
#define FP8BS_H

#include <stddef.h>
#include <stdint.h>

#if defined(FP8BS_BUILD) && defined(__GNUC__)
#define FP8BS_API __attribute__((visibility("default")))
#else
#define FP8BS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp8bs_status {
    FP8BS_OK = 0,
    FP8BS_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or shape; nothing launched */
    FP8BS_ERR_UNSUPPORTED = 2, /* well-formed but not implemented (e.g. block = 48)      */
    FP8BS_ERR_WORKSPACE = 3,   /* workspace missing or smaller than *_workspace_size()   */
    FP8BS_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed                      */
    FP8BS_ERR_TIMEOUT = 5,     /* a device-side bounded wait gave up (device error word) */
    FP8BS_ERR_SCALE = 6        /* a *_ue8m0 GEMM met a scale that is not a positive normal
                                  power of two (device error word)                        */
} fp8bs_status;

typedef enum fp8bs_dtype {
    FP8BS_DTYPE_BF16 = 0,
    FP8BS_DTYPE_F32 = 1
} fp8bs_dtype;

typedef enum fp8bs_scale_fmt {
    FP8BS_SCALE_FMT_NONE = 0,  /* s = max(amax, 1e-4) / 448 as an fp32 value         */
    FP8BS_SCALE_FMT_UE8M0 = 1  /* the same s rounded up to a power of two (exactly)   */
} fp8bs_scale_fmt;

/* Version of this ABI: major * 10000 + minor * 100 + patch. */
FP8BS_API int fp8bs_version(void);

/* Human-readable name of a status code (static storage). */
FP8BS_API const char *fp8bs_status_string(fp8bs_status status);

/* Message describing the last non-OK status returned on this host thread
 * (thread-local storage; empty string if none). */
FP8BS_API const char *fp8bs_last_error_message(void);

/* Synchronizes `stream`, then reads and clears the device error word of the
 * current device into *code (FP8BS_OK when no kernel reported a failure).
 * Returns FP8BS_ERR_CUDA if the synchronization itself failed. */
FP8BS_API fp8bs_status fp8bs_get_device_error(void *stream, int *code);

/*
 * act_quant [ACT]: dynamic 1 x block activation quantization.
 *
 * For every row r and block b of `block` consecutive elements of the last
 * dimension:
 *   amax = max |x[r, b*block + k]|               (in fp32; bf16 widens exactly)
 *   s[r, b] = max(amax, 1e-4f) / 448.0f          (IEEE fp32 division)
 *   if fmt == UE8M0: s[r, b] = smallest power of two >= s[r, b]
 *   q[r, b*block + k] = e4m3fn_rne_satfinite(x / s[r, b])   (IEEE fp32 division)
 *
 *   x      device, [rows, cols], bf16 (x_dtype = BF16) or fp32 (F32)
 *   q      device, [rows, cols], e4m3fn codes (uint8), written
 *   s      device, [rows, cols / block], fp32, written
 * cols must be a multiple of block.  block is 128 in the pages' layers and
 * is configurable ([DEQ] "Per-Block Scaling Architecture": block_size is a
 * parameter); 32, 64, 128 and 256 are implemented, other sizes return
 * FP8BS_ERR_UNSUPPORTED.  rows == 0 is a no-op.  Results are bit-exact with
 * the definition above.
 */
FP8BS_API fp8bs_status fp8bs_act_quant(const void *x, fp8bs_dtype x_dtype, int64_t rows, int64_t cols,
                             int64_t block, fp8bs_scale_fmt fmt, uint8_t *q, float *s,
                             void *stream);

/*
 * weight_dequant [DEQ]: y[i, j] = round(dec(q[i, j]) * s[i / block, j / block])
 * with the product taken in fp32 and rounded to the output type
 * (round-to-nearest-even for bf16).
 *
 *   q      device, [M, N] e4m3fn codes (uint8)
 *   s      device, [cdiv(M, block), cdiv(N, block)] fp32, row-major, so the
 *          scale of block (bi, bj) sits at bi * cdiv(N, block) + bj
 *   y      device, [M, N], bf16 (y_dtype = BF16) or fp32 (F32), written
 * Ragged M and N are allowed (edge blocks are partial).  block is 32, 64,
 * 128 or 256 (else FP8BS_ERR_UNSUPPORTED).
 * M == 0 or N == 0 is a no-op.  Bit-exact with the definition above.
 */
FP8BS_API fp8bs_status fp8bs_weight_dequant(const uint8_t *q, const float *s, int64_t M, int64_t N,
                                  int64_t block, void *y, fp8bs_dtype y_dtype, void *stream);

/*
 * act_quant_static: the static activation scheme ([STATIC]): the scales were
 * fixed ahead of time (by calibration) and ship with the checkpoint, so no
 * amax is taken; each element is divided by its block's given scale:
 *   q[r, c] = e4m3fn_rne_satfinite(x[r, c] / s[r * s_row_stride + c / block])
 * (IEEE fp32 division).  Values beyond 448 * s saturate to +-448, which the
 * dynamic scheme never needs.
 *   x            device, [rows, cols], bf16 or fp32; cols % block == 0
 *   s            device fp32 scales (4-byte aligned): s_row_stride = 0 is one
 *                scale per block of channels, [cols / block], shared by
 *                every row (the static scheme); s_row_stride >= cols / block
 *                is a per-row table with that row pitch (act_quant's s layout
 *                when equal to cols / block)
 *   q            device, [rows, cols] uint8, written
 *   s_out        device, [rows, cols / block] fp32 or NULL: when given, the
 *                scale of every (row, block) is written there, the per-row
 *                table fp8_gemm reads as a_s
 * block is 32, 64, 128 or 256 (else FP8BS_ERR_UNSUPPORTED).  Errors
 * (FP8BS_ERR_INVALID_ARG, nothing launched): cols not a positive multiple of
 * block, a stride between 0 and cols / block, an unknown dtype, null or
 * misaligned pointers, rows * cols / 16 at or above about 2^32.  rows == 0 is
 * a no-op.  A scale that is zero, negative, infinite or NaN is not an error:
 * the division and the saturating cast then give what IEEE arithmetic gives
 * (zero scale: +-448 or NaN for 0 / 0).
 */
FP8BS_API fp8bs_status fp8bs_act_quant_static(const void *x, fp8bs_dtype x_dtype, int64_t rows,
                                              int64_t cols, int64_t block, const float *s,
                                              int64_t s_row_stride, uint8_t *q, float *s_out,
                                              void *stream);

/*
 * act_dequant: static_dequant of [STATIC], the inverse of act_quant_static
 * (and, with a per-row table, of act_quant):
 *   y[r, c] = decode(q[r, c]) * s[r * s_row_stride + c / block]
 * with the product in fp32, stored as bf16 (round to nearest even) or fp32.
 *   q            device, [rows, cols] uint8 e4m3fn codes; cols % block == 0
 *   s, s_row_stride, block: as for fp8bs_act_quant_static
 *   y            device, [rows, cols], bf16 (y_dtype = BF16) or fp32, written
 * Errors as for fp8bs_act_quant_static.
 */
FP8BS_API fp8bs_status fp8bs_act_dequant(const uint8_t *q, const float *s, int64_t s_row_stride,
                                         int64_t rows, int64_t cols, int64_t block, void *y,
                                         fp8bs_dtype y_dtype, void *stream);

/*
 * weight_quant: the inverse of weight_dequant, block x block quantization of
 * a dense weight with the act_quant scale rule applied per tile:
 *   s[bi, bj] = max(amax_tile, 1e-4f) / 448.0f (optionally rounded up to 2^k)
 *   q[i, j]   = e4m3fn_rne_satfinite(w[i, j] / s[i / block, j / block])
 *   w      device, [M, N], bf16 or fp32
 *   q      device, [M, N] uint8, written;  s  device, [cdiv(M,block), cdiv(N,block)] fp32, written
 * block is 32, 64, 128 (the pages' weight_block_size) or 256.
 * Ragged M and N are allowed.  The pages state the per-tile scale layout that
 * weight_dequant consumes ([DEQ] "Per-Block Scaling Architecture"); they do
 * not print the offline quantizer, whose rule is read here as the activation
 * rule applied per 128 x 128 tile.
 */
FP8BS_API fp8bs_status fp8bs_weight_quant(const void *w, fp8bs_dtype w_dtype, int64_t M, int64_t N,
                                int64_t block, fp8bs_scale_fmt fmt, uint8_t *q, float *s,
                                void *stream);

/*
 * fp8_gemm [GEMM]: y = A * W^T on block-scaled FP8 operands, FP32
 * accumulation, bf16 output:
 *   y[m, n] = bf16( sum_kb a_s[m, kb] * w_s[n / 128, kb] * P_kb[m, n] ),
 *   P_kb[m, n] = sum_{k in kb} dec(a[m, k]) * dec(w[n, k]),   kb = k / 128.
 *
 *   a      device, [M, K] e4m3fn codes
 *   a_s    device, [M, K / 128] fp32 (the layout act_quant writes)
 *   w      device, [N, K] e4m3fn codes (the nn.Linear weight layout)
 *   w_s    device, [cdiv(N, 128), K / 128] fp32 (the layout weight_dequant reads)
 *   y      device, [M, N] bf16, written
 *   workspace / workspace_bytes: device scratch of at least
 *          fp8bs_gemm_workspace_size(M, N, K) bytes (may be NULL when that is 0);
 *          its contents on entry do not matter.
 * K must be a positive multiple of 128.  M and N may be ragged.  M == 0 or
 * N == 0 is a no-op.  Results are within |dy| <= 4e-3 |y_ref| +
 * 1e-3 sum_k |a_hat_k w_hat_k| of the exact value y_ref.
 */
FP8BS_API size_t fp8bs_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * Self-test of the division act_quant uses for scale_fmt NONE: q[i] =
 * x[i] / s[i] by Markstein's division correction from RN(1/s).  q[i] is the
 * correctly rounded fp32 quotient whenever |x[i]| and |x[i]/s[i]| are at
 * least 2^-100 (nothing in the correction underflows); below that it may be
 * off by ulps of a value far under the smallest e4m3 step, which rounds to
 * the same e4m3 code.  x, s, q are device fp32 arrays of n elements, s[i] a
 * positive normal number.  For verification only.
 */
FP8BS_API fp8bs_status fp8bs_selftest_quotient(const float *x, const float *s, float *q, int64_t n,
                                               void *stream);

/*
 * Self-test of the per-block scale rule that act_quant and weight_quant
 * apply to a block's absolute maximum ([ACT]; scale_fmt as in act_quant):
 * s[i] = max(amax[i], 1e-4) / 448 as the correctly rounded fp32 quotient,
 * then for FP8BS_SCALE_FMT_UE8M0 the smallest power of two >= that.  amax and s
 * are device fp32 arrays of n elements; amax[i] is a non-negative number or
 * +inf.  Errors: FP8BS_ERR_INVALID_ARG for n < 0, a null pointer with n > 0
 * or an unknown scale_fmt.  For verification only.
 */
FP8BS_API fp8bs_status fp8bs_selftest_block_scale(const float *amax, float *s, int64_t n,
                                                  int scale_fmt, void *stream);

/*
 * Self-test of the GEMM's bounded device waits (the pages show no failure
 * handling; this is the library's own failure path).  Runs fp8bs_fp8_gemm
 * with one arrival withheld: the first CTA's scale producer does not signal
 * its K-block step stall_step - 1 (counted over that CTA's work units from
 * 0), so the epilogue's wait for that step cannot complete.  The wait gives
 * up after its limit (about 2 s), records FP8BS_ERR_TIMEOUT in the device
 * error word, and every role of that CTA drains the copies and MMAs it has in
 * flight, releases its tensor memory and exits; the other CTAs finish
 * normally.  The context stays usable: fp8bs_get_device_error() then returns
 * FP8BS_ERR_TIMEOUT, and later calls run normally.  y is left partly
 * unwritten.  Arguments as for fp8bs_fp8_gemm, plus stall_step >= 1 (else
 * FP8BS_ERR_INVALID_ARG); a step past the CTA's last one withholds nothing.
 * For verification only.
 */
FP8BS_API fp8bs_status fp8bs_selftest_gemm_stall(const uint8_t *a, const float *a_s,
                                                 const uint8_t *w, const float *w_s, int64_t M,
                                                 int64_t N, int64_t K, uint16_t *y,
                                                 void *workspace, size_t workspace_bytes,
                                                 int stall_step, void *stream);

/* Launch plan fp8_gemm would use for an M x N x K problem on the current
 * device (tile width, K split, work units, grid), as a
 * NUL-terminated string in thread-local storage; for logs and benchmarks. */
FP8BS_API const char *fp8bs_gemm_plan_string(int64_t M, int64_t N, int64_t K);

FP8BS_API fp8bs_status fp8bs_fp8_gemm(const uint8_t *a, const float *a_s, const uint8_t *w,
                            const float *w_s, int64_t M, int64_t N, int64_t K, uint16_t *y,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * fp8_gemm for callers that cannot allocate device memory.  (The pages have
 * no counterpart: this entry point is an addition for deployment.)
 *
 * Some callers cannot call cudaMalloc at the time of the call, or cannot own
 * a scratch buffer at all: for example an inference server that reserves its
 * whole device memory budget at start-up and forbids later allocations, a
 * plugin inside a host framework that owns the allocator, or a plain C caller
 * that has no allocator for a workspace.  This entry point computes exactly
 * what fp8bs_fp8_gemm computes, and allocates nothing: the split-K partials
 * that fp8bs_fp8_gemm would keep in the caller's workspace go to a scratch
 * array of FP8BS_STATIC_SCRATCH_BYTES that the library holds in device
 * memory on every GPU that loads it, until the process exits.
 *
 *   a, a_s, w, w_s, y, M, N, K: as for fp8bs_fp8_gemm (caller-owned device
 *   buffers; inputs and output are still the caller's).
 *
 * Problems whose plan needs more split-K scratch than
 * FP8BS_STATIC_SCRATCH_BYTES (fp8bs_gemm_workspace_size(M, N, K) is larger)
 * are rejected with FP8BS_ERR_WORKSPACE before anything is launched.
 *
 * An empty problem (M == 0) is validated like fp8bs_fp8_gemm and returns
 * FP8BS_OK without touching the device.  The first call with M > 0 on a
 * device looks up the scratch array's device address (cudaGetSymbolAddress,
 * once per device, on the current device) and keeps it for the life of the
 * process (invalid after cudaDeviceReset(), as all per-device set-up above);
 * make that first call before any stream capture.  All calls share the one array and
 * every call writes the partials it reads, so nothing needs clearing between
 * calls, but calls that overlap on the GPU (other streams, other threads)
 * race on the array: serialise them.
 */
#define FP8BS_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

FP8BS_API fp8bs_status fp8bs_fp8_gemm_static_scratch(const uint8_t *a, const float *a_s,
                                                     const uint8_t *w, const float *w_s,
                                                     int64_t M, int64_t N, int64_t K,
                                                     uint16_t *y, void *stream);

/*
 * fp8_gemm_ue8m0: fp8_gemm for power-of-two scales ([ACT]: scale_fmt "ue8m0"
 * rounds scales to powers of two for hardware compatibility).  Same
 * arguments, layouts, workspace and result as fp8bs_fp8_gemm, but every a_s
 * and w_s entry must be a positive normal power of two, which the tensor core
 * then applies itself (tcgen05.mma kind::mxf8f6f4.block_scale with ue8m0
 * scale factors, one FP32 accumulation over all of K).  Decode-sized M (up
 * to 64 rows), where the weight stream decides the time, runs the
 * per-K-block promotion kernel instead, which is faster there and gives a
 * result within the same tolerance.  On either path a scale that is not
 * such a power of two is reported through the device error word
 * (FP8BS_ERR_SCALE) and makes the output meaningless.
 */
FP8BS_API fp8bs_status fp8bs_fp8_gemm_ue8m0(const uint8_t *a, const float *a_s, const uint8_t *w,
                                            const float *w_s, int64_t M, int64_t N, int64_t K,
                                            uint16_t *y, void *workspace, size_t workspace_bytes,
                                            void *stream);

/*
 * fp8_gemm_f32: fp8_gemm with an FP32 output ("DeepSeek-V3: How Selective FP8
 * Stays Stable", "Lower precision is a constrained budget": the FP8 GEMMs'
 * outputs may be BF16 or FP32).  The same product as fp8bs_fp8_gemm, stored
 * as the FP32 accumulator without the final rounding to bf16.
 *
 *   a, a_s, w, w_s, M, N, K, workspace: as for fp8bs_fp8_gemm (the same
 *     fp8bs_gemm_workspace_size(M, N, K) bytes suffice);
 *   fmt   FP8BS_SCALE_FMT_NONE: any positive fp32 scales (per-K-block
 *         promotion, as fp8bs_fp8_gemm); FP8BS_SCALE_FMT_UE8M0: every scale a
 *         positive normal power of two (block-scaled MMA, as
 *         fp8bs_fp8_gemm_ue8m0, with the same FP8BS_ERR_SCALE report);
 *         anything else is FP8BS_ERR_INVALID_ARG;
 *   y     device, [M, N] fp32, written (16-byte aligned).
 */
FP8BS_API fp8bs_status fp8bs_fp8_gemm_f32(const uint8_t *a, const float *a_s, const uint8_t *w,
                                          const float *w_s, int64_t M, int64_t N, int64_t K,
                                          fp8bs_scale_fmt fmt, float *y, void *workspace,
                                          size_t workspace_bytes, void *stream);

/*
 * act_quant_transposed: quantization in block x 1 column blocks, written
 * transposed ([TRAIN]): the K-major operand layout of the weight-gradient
 * GEMM, which contracts over the rows of x (the tokens).  By definition
 *   (qt, st) = act_quant(x^T, block, fmt)
 * i.e. for column c and row block rb the amax of x[rb*block .. +block, c],
 * the act_quant scale rule, and qt[c, r] = e4m3fn_rne_satfinite(x[r, c] / s).
 *   x      device, [rows, cols], bf16 or fp32; rows % block == 0 (else
 *          FP8BS_ERR_INVALID_ARG), cols % 8 == 0 (else FP8BS_ERR_UNSUPPORTED)
 *   qt     device, [cols, rows] uint8, written
 *   st     device, [cols, rows / block] fp32, written
 * block is 128 (others: FP8BS_ERR_UNSUPPORTED).  rows == 0 is a no-op.
 */
FP8BS_API fp8bs_status fp8bs_act_quant_transposed(const void *x, fp8bs_dtype x_dtype,
                                                  int64_t rows, int64_t cols, int64_t block,
                                                  fp8bs_scale_fmt fmt, uint8_t *qt, float *st,
                                                  void *stream);

/*
 * fp8_transpose: the transposed FP8 matrix and its transposed block scales,
 * exactly ([TRAIN]: the activation-gradient GEMM dx = dy W contracts over W's
 * rows, so it runs as fp8_gemm(dy, W^T)):
 *   qt[c, r] = q[r, c],  st[j, i] = s[i, j]
 *   q      device, [R, C] uint8;  s  device, [cdiv(R,block), cdiv(C,block)] fp32
 *   qt     device, [C, R] uint8, written (not aliasing q)
 *   st     device, [cdiv(C,block), cdiv(R,block)] fp32, written
 * block (32, 64, 128 or 256) only sizes the scale tables.  Any R and C; the
 * tiled path needs R and C multiples of 16, other shapes take a slower
 * element-wise kernel.
 */
FP8BS_API fp8bs_status fp8bs_fp8_transpose(const uint8_t *q, const float *s, int64_t R,
                                           int64_t C, int64_t block, uint8_t *qt, float *st,
                                           void *stream);

/*
 * fp8_gemm_rowwise: the GEMM whose two operands both carry one scale per row
 * and 128-wide K block, the form of the weight-gradient GEMM of a linear
 * layer ([TRAIN]: all three GEMMs of a linear layer run in FP8, and weight
 * gradients stay FP32):
 *   y[m, n] = sum_kb a_s[m, kb] * b_s[n, kb] * sum_{k in kb} a[m, k] * b[n, k]
 * For dW = dy^T x over T tokens: a = dy^T and b = x^T, both quantized in
 * 128 x 1 blocks along the tokens, as fp8bs_act_quant_transposed writes them
 * (a: [N_out, T], b: [K_in, T], K = T).
 *   a      device, [M, K] e4m3fn codes;  a_s  device, [M, K / 128] fp32
 *   b      device, [N, K] e4m3fn codes;  b_s  device, [N, K / 128] fp32
 *   fmt    FP8BS_SCALE_FMT_NONE (any positive fp32 scales: per-K-block FP32
 *          promotion with a scale per column) or FP8BS_SCALE_FMT_UE8M0 (all
 *          scales positive normal powers of two: the block-scaled MMA, with
 *          the FP8BS_ERR_SCALE report of fp8bs_fp8_gemm_ue8m0)
 *   y      device, [M, N], fp32 (y_dtype = F32) or bf16, written
 *   workspace: fp8bs_gemm_rowwise_workspace_size(M, N, K) bytes (the split-K
 *          partials and K-block-major copies of a_s and b_s, which make the
 *          kernels' scale loads coalesced)
 * K % 128 == 0, ragged M and N; errors as for fp8bs_fp8_gemm, plus
 * FP8BS_ERR_INVALID_ARG for an unknown fmt or y_dtype.
 */
FP8BS_API size_t fp8bs_gemm_rowwise_workspace_size(int64_t M, int64_t N, int64_t K);

FP8BS_API fp8bs_status fp8bs_fp8_gemm_rowwise(const uint8_t *a, const float *a_s,
                                              const uint8_t *b, const float *b_s, int64_t M,
                                              int64_t N, int64_t K, fp8bs_scale_fmt fmt, void *y,
                                              fp8bs_dtype y_dtype, void *workspace,
                                              size_t workspace_bytes, void *stream);

/*
 * fp8_linear_ue8m0: act_quant(x, 128, UE8M0) followed by fp8_gemm_ue8m0 on
 * one stream.  Arguments as for fp8bs_fp8_linear; w_s must hold powers of
 * two (weights quantized with the ue8m0 scale format).
 */
FP8BS_API fp8bs_status fp8bs_fp8_linear_ue8m0(const uint16_t *x, int64_t M, int64_t K,
                                              const uint8_t *w, const float *w_s, int64_t N,
                                              uint16_t *y, uint8_t *q, float *s, void *workspace,
                                              size_t workspace_bytes, void *stream);

/*
 * fp8_linear: the FP8 linear layer's forward pass ([ACT] notes that the
 * linear wrapper calls act_quant during the forward pass):
 *   (q, s) = act_quant(x, 128, fmt);  y = fp8_gemm(q, s, w, w_s)
 *
 *   x      device, [M, K] bf16 (16-byte aligned)
 *   w, w_s as for fp8_gemm;  y  device, [M, N] bf16, written
 *   q      device, [M, K] uint8 and  s  device, [M, K / 128] fp32: caller-
 *          provided buffers that receive the quantized activations and scales
 *          (bit for bit what fp8bs_act_quant writes)
 *   workspace  fp8bs_linear_workspace_size(M, N, K) bytes (16-byte aligned)
 *
 * Two forms, chosen per shape by their estimated times
 * (fp8bs_linear_plan_string says which):
 *  - act_quant followed by fp8_gemm, two launches on the stream (the
 *    workspace then serves fp8_gemm, as fp8bs_gemm_workspace_size says);
 *  - the single fused launch of fp8bs_fp8_linear_fused (below), taken only
 *    where its estimate is lower.  With the costs measured on B200 it is
 *    slower at every prefill shape measured, so the two launches are taken.
 * q, s and y are the same in both forms (the GEMM's tile plan may differ, so
 * y may differ in the last bits within the GEMM tolerance).
 */
FP8BS_API fp8bs_status fp8bs_fp8_linear(const uint16_t *x, int64_t M, int64_t K, fp8bs_scale_fmt fmt,
                              const uint8_t *w, const float *w_s, int64_t N, uint16_t *y,
                              uint8_t *q, float *s, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * fp8_linear_fused: the same layer as fp8bs_fp8_linear in ONE kernel launch
 * (plus a memset of the workspace flags before it).  Where the GEMM's output
 * tiles leave SMs idle (narrow N at M > 128, e.g. M = 4096, N = 576), those
 * SMs quantize x while the others run the GEMM a few K blocks behind: every
 * quantized 128-row chunk of a K block is counted into a flag in the
 * workspace (release at GPU scope), and a GEMM CTA reads a chunk's codes and
 * scales only after its flag (acquire).  Each chunk is quantized once, by the
 * same arithmetic as act_quant, so q and s are bit-identical to
 * fp8bs_act_quant's.  Useful where one launch matters more than time (a
 * stream with a fixed kernel count); on B200 it measured slower than the two
 * launches at the prefill shapes (the idle SMs quantize at ~35 GB/s each).
 *
 *   arguments as for fp8bs_fp8_linear; the workspace needs 4 bytes per
 *   (128-row tile, K block), which fp8bs_linear_workspace_size covers.
 * Errors: FP8BS_ERR_UNSUPPORTED when M <= 128 or the tiles leave fewer than
 * 16 SMs free (no fused launch exists), FP8BS_ERR_WORKSPACE for a short
 * workspace, and the checks of fp8bs_fp8_linear.
 */
FP8BS_API fp8bs_status fp8bs_fp8_linear_fused(const uint16_t *x, int64_t M, int64_t K,
                                              fp8bs_scale_fmt fmt, const uint8_t *w,
                                              const float *w_s, int64_t N, uint16_t *y,
                                              uint8_t *q, float *s, void *workspace,
                                              size_t workspace_bytes, void *stream);

/* Workspace bytes fp8bs_fp8_linear and fp8bs_fp8_linear_fused need on the
 * current device for an M x N x K layer (0 for invalid sizes). */
FP8BS_API size_t fp8bs_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/* Which form fp8bs_fp8_linear takes for an M x N x K layer on the current
 * device, and its tile plan, as a NUL-terminated string in thread-local
 * storage; for logs and benchmarks. */
FP8BS_API const char *fp8bs_linear_plan_string(int64_t M, int64_t N, int64_t K);

/*
 * fp8_gemm_grouped: G independent fp8_gemm problems (experts) that share N
 * and K, with the rows of A grouped contiguously by problem:
 *   rows m_offsets[g] .. m_offsets[g+1]-1 of a / a_s / y belong to problem g,
 *   y[rows of g] = fp8_gemm(a[rows of g], a_s[rows of g], w[g], w_s[g]).
 *
 *   m_offsets   DEVICE, G + 1 int64 prefix offsets (m_offsets[0] = 0,
 *               non-decreasing, m_offsets[G] <= M_total); the host never reads
 *               them, so routing results need no host synchronization.  A group
 *               whose end is below its start is empty; rows outside
 *               [0, M_total) are never read or written.  Offsets that
 *               decrease break the contract: memory stays safe (each group is
 *               clamped to [0, M_total)), but a later group may then overlap
 *               an earlier group's rows, whose y is then unspecified.
 *   a      device, [M_total, K];  a_s  device, [M_total, K / 128]
 *   w      device, [G, N, K];     w_s  device, [G, cdiv(N, 128), K / 128]
 *   y      device, [M_total, N] bf16; rows that belong to no group are left
 *          untouched.
 * 1 <= G <= 1024.  Same K constraint and tolerance as fp8_gemm.  Needs no
 * workspace.
 */
FP8BS_API fp8bs_status fp8bs_fp8_gemm_grouped(int64_t G, const int64_t *m_offsets, int64_t M_total,
                                    const uint8_t *a, const float *a_s, const uint8_t *w,
                                    const float *w_s, int64_t N, int64_t K, uint16_t *y,
                                    void *stream);

/*
 * fp8_gemm_grouped_ue8m0: fp8_gemm_grouped with the power-of-two scale
 * requirement and the block-scaled MMA of fp8_gemm_ue8m0.  Same arguments.
 */
FP8BS_API fp8bs_status fp8bs_fp8_gemm_grouped_ue8m0(int64_t G, const int64_t *m_offsets,
                                                    int64_t M_total, const uint8_t *a,
                                                    const float *a_s, const uint8_t *w,
                                                    const float *w_s, int64_t N, int64_t K,
                                                    uint16_t *y, void *stream);

/*
 * fp8_gemm_quant: fp8_gemm with an FP8 output, for a following FP8 linear.
 * The product y = a * w^T (same operands, layouts, constraints and
 * tolerance as fp8_gemm, any fp32 scales) is rounded to bf16 and quantized
 * exactly as fp8bs_act_quant(y_bf16, block = 128, out_fmt) would quantize it:
 * per 1x128 block of each output row, s = max(amax, 1e-4) / 448 (ue8m0:
 * the next power of two up), q = e4m3(y / s).  This is the "fuse the
 * activation quantization into the producing GEMM's epilogue" step that the
 * pages' linear layer leaves to a separate act_quant call ("Understanding
 * Dynamic and Static Activation Quantization Schemes in DeepSeek-V3", "How
 * Dynamic Activation Quantization Works"; the fused form has no counterpart on
 * the pages and is checked bit for bit against fp8bs_act_quant of the bf16 y).
 *   q_out  device, [M, N] uint8 (e4m3fn codes), 16-byte aligned
 *   s_out  device, [M, N / 128] float32
 *   y      device, [M, N] bf16, or NULL; when given it receives the bf16 y
 *          that q_out and s_out quantize.
 * N % 128 == 0 (else FP8BS_ERR_INVALID_ARG).  Needs no workspace.  Runs the
 * promotion kernel with 128 x 256 tiles and no K split.
 */
FP8BS_API fp8bs_status fp8bs_fp8_gemm_quant(const uint8_t *a, const float *a_s, const uint8_t *w,
                                            const float *w_s, int64_t M, int64_t N, int64_t K,
                                            fp8bs_scale_fmt out_fmt, uint8_t *q_out, float *s_out,
                                            uint16_t *y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8BS_H */
