/*
 * CPU oracle for the FP8 block-scaled linear-layer path of DeepSeek-V3:
 * dynamic 1x128 activation quantization, 128x128-block weight
 * dequantization, and the block-scaled FP8 GEMM y = A * W^T.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA path computes.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant generator with the CUDA library, and the CUDA
 * library never calls it.
 *
 * Sources (page title, then section):
 *  [P1] "Understanding Dynamic and Static Activation Quantization Schemes in
 *       DeepSeek-V3", section "How Dynamic Activation Quantization Works":
 *       block of 128 channels, s = amax / 448 with amax clamped, optional
 *       power-of-two scales for scale_fmt "ue8m0"; section "Frequently Asked
 *       Questions": e4m3fn has 4 exponent and 3 mantissa bits.
 *  [P2] "DeepSeek-V3 quantization_config Parameters Explained: e4m3,
 *       weight_block_size, and activation_scheme", section "The
 *       activation_scheme Parameter": amax of each block clamped to a minimum
 *       of 1e-4, s = amax / 448, 448 the largest e4m3 value; section "The fmt
 *       Parameter": the quantized dtype is torch.float8_e4m3fn; section "The
 *       weight_block_size Parameter": one scale per 128x128 weight block,
 *       multiplied in (y = x * s).
 *  [P4] "How weight_dequant Handles Per-Block Scaling in DeepSeek-V3 FP8
 *       GEMM", section "Grid Mapping and Scale Lookup": the scale of block
 *       (pid_m, pid_n) sits at pid_m * cdiv(N, 128) + pid_n; section
 *       "Dequantization Computation": fp32 value = fp8 value * block scale,
 *       masked at the edges; section "Relationship to FP8 GEMM Operations":
 *       fp8_gemm(a, a_s, b, b_s) applies the same per-block scales inside the
 *       matrix product.
 *  [P5] "DeepSeek-V3: How Selective FP8 Stays Stable", section "Learning
 *       outcomes": 1x128 activation tiles, 128x128 weight blocks, partial sums
 *       promoted to FP32.
 *  The bit layout of e4m3fn (exponent bias 7, no infinities, NaN = S.1111.111,
 *  smallest subnormal 2^-9) is the OCP 8-bit floating point format that
 *  torch.float8_e4m3fn implements; the pages name the dtype but not its bits.
 *
 * Readings where the pages leave a step open (each is listed in the design
 * notes): the amax is taken per 1x128 block, not per row; the clamp is the
 * fp32 value of 1e-4 applied before the division; q = x / s is an IEEE fp32
 * division followed by a round-to-nearest-even, saturating cast to e4m3fn;
 * "ue8m0" rounds s up to the next power of two (exactly); weight scales have
 * cdiv(rows,128) x cdiv(cols,128) entries; weight_dequant rounds the fp32
 * product to bf16 with round-to-nearest-even.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * The floating point here is plain C on x86-64 SSE: float arithmetic is IEEE
 * binary32 with round-to-nearest-even, double is binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <omp.h>

/* ------------------------------------------------------------------------ */
/* e4m3fn codec, written from the format definition.                          */
/* ------------------------------------------------------------------------ */

/* Value of an e4m3fn code.  Layout S EEEE MMM, exponent bias 7.
 * E == 0 is subnormal (M * 2^-9); E == 15 with M == 7 is NaN; there is no
 * infinity, so E == 15, M < 7 are ordinary numbers up to 1.75 * 2^8 = 448. */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return sign ? -NAN : NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                 /* m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round-to-nearest-even cast of an fp32 value to e4m3fn with saturation to
 * the largest finite value (+-448); NaN keeps its sign and becomes S.1111.111.
 * All arithmetic here is exact in double: a is an fp32 value and the quantum
 * is a power of two. */
uint8_t oracle_e4m3_encode(float f)
{
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a, quantum, v;
    int e, E;

    if (isnan(f))
        return sign | 0x7F;
    a = fabs((double)f);
    if (a >= 448.0)                               /* includes +-inf */
        return sign | 0x7E;

    /* Grid spacing of e4m3 around a: 3 fraction bits in binade [2^E, 2^E+1),
     * and the subnormal range shares the spacing of the lowest binade E=-6. */
    if (a == 0.0) {
        E = -6;
    } else {
        frexp(a, &e);                             /* a in [2^(e-1), 2^e) */
        E = e - 1;
        if (E < -6)
            E = -6;
    }
    quantum = ldexp(1.0, E - 3);
    v = rint(a / quantum) * quantum;              /* ties go to the even multiple */

    if (v == 0.0)
        return sign;
    frexp(v, &e);
    E = e - 1;
    if (E < -6)                                   /* subnormal code: v = M * 2^-9 */
        return sign | (uint8_t)(v / ldexp(1.0, -9));
    return sign | (uint8_t)(((E + 7) << 3) | (int)((v / ldexp(1.0, E) - 1.0) * 8.0));
}

/* Element-wise encode of n fp32 values (a loop over the scalar codec). */
void oracle_e4m3_encode_array(const float *f, int64_t n, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_e4m3_encode(f[i]);
}

/* ------------------------------------------------------------------------ */
/* bfloat16 conversions.                                                       */
/* ------------------------------------------------------------------------ */

/* bf16 keeps the top 16 bits of the fp32 pattern; the widening is exact. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round-to-nearest-even narrowing of fp32 to bf16: drop the low 16 bits of
 * the pattern, rounding up when they exceed half, or equal half and the kept
 * part is odd.  A carry out of the fraction correctly bumps the exponent (up
 * to infinity).  NaN stays NaN (quiet bit set, sign kept). */
uint16_t oracle_bf16_from_f32(float f)
{
    uint32_t u, kept, rest;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    kept = u >> 16;
    rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (kept & 1u)))
        kept += 1;
    return (uint16_t)kept;
}

/* ------------------------------------------------------------------------ */
/* Scale rule shared by the activation quantizer and the test-data weight     */
/* quantizer: s = max(amax, 1e-4) / 448, optionally rounded up to 2^k.        */
/* ------------------------------------------------------------------------ */

/* Smallest power of two >= s, for finite s > 0 (exact: frexp/ldexp). */
float oracle_ue8m0_round_up(float s)
{
    int e;
    double f;
    if (!isfinite(s))                             /* +inf: no larger power of two */
        return s;
    f = frexp((double)s, &e);                     /* s = f * 2^e, f in [0.5, 1) */
    if (f == 0.5)
        return s;
    return (float)ldexp(1.0, e);
}

/* [P2 "The activation_scheme Parameter"] clamp then divide by 448 (fp32);
 * [P1 "How Dynamic Activation Quantization Works"] "ue8m0" power-of-two. */
float oracle_block_scale(float amax, int ue8m0)
{
    float a = amax > 1e-4f ? amax : 1e-4f;
    float s = a / 448.0f;
    if (ue8m0)
        s = oracle_ue8m0_round_up(s);
    return s;
}

/* ------------------------------------------------------------------------ */
/* act_quant: one scale per 1 x block run of the last dimension.             */
/* x is [rows, cols] row-major, bf16 (x_is_bf16 = 1) or fp32; cols % block    */
/* must be 0 (the caller checks).  q is [rows, cols], s is [rows, cols/block].*/
/* ------------------------------------------------------------------------ */

static float load_x(const void *x, int x_is_bf16, int64_t i)
{
    if (x_is_bf16)
        return oracle_bf16_to_f32(((const uint16_t *)x)[i]);
    return ((const float *)x)[i];
}

void oracle_act_quant(const void *x, int x_is_bf16, int64_t rows, int64_t cols,
                      int64_t block, int ue8m0, uint8_t *q, float *s)
{
    int64_t nblk = cols / block;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nblk; b++) {
            int64_t base = r * cols + b * block;
            float amax = 0.0f, sc;
            for (int64_t k = 0; k < block; k++) {
                float v = fabsf(load_x(x, x_is_bf16, base + k));
                if (v > amax)
                    amax = v;
            }
            sc = oracle_block_scale(amax, ue8m0);
            s[r * nblk + b] = sc;
            for (int64_t k = 0; k < block; k++)
                q[base + k] = oracle_e4m3_encode(load_x(x, x_is_bf16, base + k) / sc);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Static activation scheme [P1 "How Static Activation Quantization          */
/* Differs"]: the scales are fixed ahead of time (from calibration) and      */
/* stored with the checkpoint, so no amax is taken.  The scale of element    */
/* (r, c) is s[r * s_row_stride + c / block]: s_row_stride = 0 is one scale   */
/* per block of channels shared by every row (the static scheme); a stride of */
/* cols / block is a per-row scale table such as act_quant writes.  Each code */
/* is the same rule as in act_quant without the scale step:                   */
/* q = encode(fl32(x / s)), IEEE fp32 division, then the round-to-nearest-    */
/* even, saturating cast, which now can saturate (|x| may exceed 448 s).      */
/* ------------------------------------------------------------------------ */

void oracle_act_quant_static(const void *x, int x_is_bf16, int64_t rows, int64_t cols,
                             int64_t block, const float *s, int64_t s_row_stride, uint8_t *q)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float sc = s[r * s_row_stride + c / block];
            q[r * cols + c] = oracle_e4m3_encode(load_x(x, x_is_bf16, r * cols + c) / sc);
        }
}

/* Activation dequantization [P1 "How Static Activation Quantization         */
/* Differs", static_dequant]: value = fp8 value times its block's scale, the */
/* product in fp32 (the page multiplies q_x.float() by the scales broadcast   */
/* over each block), stored as fp32 or rounded to bf16 (RNE).  Scale lookup   */
/* as in oracle_act_quant_static.                                             */
void oracle_act_dequant(const uint8_t *q, const float *s, int64_t s_row_stride, int64_t rows,
                        int64_t cols, int64_t block, int y_is_bf16, void *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float p = (float)oracle_e4m3_decode(q[r * cols + c]) * s[r * s_row_stride + c / block];
            if (y_is_bf16)
                ((uint16_t *)y)[r * cols + c] = oracle_bf16_from_f32(p);
            else
                ((float *)y)[r * cols + c] = p;
        }
}

/* ------------------------------------------------------------------------ */
/* Test-data weight quantizer: the same scale rule over block x block tiles   */
/* of an fp32 matrix [rows, cols]; edge tiles are partial.  s has            */
/* cdiv(rows,block) x cdiv(cols,block) entries.  Not a library call: it makes */
/* the quantized weights that the GEMM tests and the CPU baseline consume.    */
/* ------------------------------------------------------------------------ */

void oracle_weight_quant(const float *w, int64_t rows, int64_t cols, int64_t block,
                         int ue8m0, uint8_t *q, float *s)
{
    int64_t rb = (rows + block - 1) / block, cb = (cols + block - 1) / block;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rb * cb; t++) {
        int64_t bi = t / cb, bj = t % cb;
        int64_t r0 = bi * block, c0 = bj * block;
        int64_t r1 = r0 + block < rows ? r0 + block : rows;
        int64_t c1 = c0 + block < cols ? c0 + block : cols;
        float amax = 0.0f, sc;
        for (int64_t r = r0; r < r1; r++)
            for (int64_t c = c0; c < c1; c++) {
                float v = fabsf(w[r * cols + c]);
                if (v > amax)
                    amax = v;
            }
        sc = oracle_block_scale(amax, ue8m0);
        s[t] = sc;
        for (int64_t r = r0; r < r1; r++)
            for (int64_t c = c0; c < c1; c++)
                q[r * cols + c] = oracle_e4m3_encode(w[r * cols + c] / sc);
    }
}

/* ------------------------------------------------------------------------ */
/* weight_dequant [P4 "Dequantization Computation"]: y = fp8 * s in fp32,     */
/* the scale of element (i, j) being s[(i/block) * cdiv(N,block) + j/block].  */
/* y_is_bf16: store the fp32 product rounded to bf16 (RNE), else fp32.        */
/* ------------------------------------------------------------------------ */

void oracle_weight_dequant(const uint8_t *q, const float *s, int64_t M, int64_t N,
                           int64_t block, int y_is_bf16, void *y)
{
    int64_t n = (N + block - 1) / block;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; i++) {
        for (int64_t j = 0; j < N; j++) {
            float v = (float)oracle_e4m3_decode(q[i * N + j]);
            float p = v * s[(i / block) * n + j / block];
            if (y_is_bf16)
                ((uint16_t *)y)[i * N + j] = oracle_bf16_from_f32(p);
            else
                ((float *)y)[i * N + j] = p;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Block-scaled FP8 GEMM reference [P4 "Relationship to FP8 GEMM             */
/* Operations"; P5 "Learning outcomes"]:                                      */
/*   y[m,n] = sum_kb sa[m,kb] * sw[n/block,kb] * P_kb[m,n],                   */
/*   P_kb[m,n] = sum_{k in kb} dec(qa[m,k]) * dec(qw[n,k]),                   */
/* with A = [M,K], W = [N,K] (y = A W^T), sa = [M, K/block],                  */
/* sw = [cdiv(N,block), K/block].  sw_rows = block gives that weight layout;  */
/* sw_rows = 1 gives one scale per row of W and K block, sw = [N, K/block],   */
/* the second operand of the weight-gradient GEMM [P5 "Lower precision is a   */
/* constrained budget": all three GEMMs of a linear layer run in FP8], whose  */
/* operands are both activations-like (quantized along the contracted dim).   */
/* P_kb is exact in double: each product is a */
/* multiple of 2^-18 below 2^18 and 128 of them need under 53 bits.  Also    */
/* returns bound[m,n] = sum_k |dec(qa)*sa * dec(qw)*sw|, the scale of the    */
/* rounding error that FP32 accumulation may make.                            */
/* Rows of A are processed in the order given; only the loops over m and n    */
/* are parallel, each y[m,n] is one sequential sum.                           */
/* ------------------------------------------------------------------------ */

void oracle_gemm(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                 int64_t M, int64_t N, int64_t K, int64_t block, int64_t sw_rows, double *y,
                 double *bound)
{
    int64_t kbn = K / block;
    double table[256];
    for (int c = 0; c < 256; c++)
        table[c] = oracle_e4m3_decode((uint8_t)c);

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; n++) {
        const uint8_t *wrow = qw + n * K;
        const float *swrow = sw + (n / sw_rows) * kbn;
        for (int64_t m = 0; m < M; m++) {
            const uint8_t *arow = qa + m * K;
            double acc = 0.0, babs = 0.0;
            for (int64_t kb = 0; kb < kbn; kb++) {
                double p = 0.0, pabs = 0.0;
                double scale = (double)sa[m * kbn + kb] * (double)swrow[kb];
                for (int64_t k = kb * block; k < (kb + 1) * block; k++) {
                    double prod = table[arow[k]] * table[wrow[k]];
                    p += prod;
                    pabs += fabs(prod);
                }
                acc += scale * p;
                babs += fabs(scale) * pabs;
            }
            y[m * N + n] = acc;
            if (bound)
                bound[m * N + n] = babs;
        }
    }
}

int oracle_num_threads(void)
{
    return omp_get_max_threads();
}
