// Streaming kernels of the FP8 block-scaled path: dynamic 1x128 activation
// quantization (act_quant), 128x128-block weight dequantization
// (weight_dequant), the per-tile weight quantizer (weight_quant) and the
// split-K reduction of the GEMM.
//
// act_quant follows "Understanding Dynamic and Static Activation Quantization
// Schemes in DeepSeek-V3", section "How Dynamic Activation Quantization
// Works", and "DeepSeek-V3 quantization_config Parameters Explained", section
// "The activation_scheme Parameter": per block of 128 channels,
// s = max(amax, 1e-4) / 448 (optionally a power of two, "ue8m0"), q = x / s
// cast to float8_e4m3fn.  weight_dequant follows "How weight_dequant Handles
// Per-Block Scaling in DeepSeek-V3 FP8 GEMM", sections "Grid Mapping and Scale
// Lookup" and "Dequantization Computation": y = fp8 * s[i/128, j/128] in fp32,
// masked at ragged edges.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace fp8bs {

// ---------------------------------------------------------------------------
// Scalar pieces
// ---------------------------------------------------------------------------

// Correctly rounded fp32 quotient x / d from r = RN(1/d) by Markstein's
// division correction (see quotient2 below for the method and its premises).
__device__ __forceinline__ float quotient1(float x, float r, float nd) {
  float q = x * r;
  q = fmaf(fmaf(q, nd, x), r, q);
  q = fmaf(fmaf(q, nd, x), r, q);
  return q;
}

// s = max(amax, 1e-4f) / 448, correctly rounded (the division by the
// constant 448 through quotient1 with r = RN(1/448), a compile-time constant;
// a >= 1e-4 keeps every step far from underflow, and an infinite amax, where
// the correction would produce inf - inf, is passed through as the quotient
// inf / 448 = inf); for ue8m0 the smallest power of two >= s, taken on the
// bit pattern (s is a positive normal number): a nonzero fraction bumps the
// exponent and clears the fraction.
__device__ __forceinline__ float block_scale(float amax, bool ue8m0) {
  const float a = fmaxf(amax, 1e-4f);
  float s = quotient1(a, 1.0f / 448.0f, -448.0f);
  if (isinf(a)) s = a;
  if (ue8m0) {
    uint32_t u = __float_as_uint(s);
    if (u & 0x007FFFFFu) u = (u & 0x7F800000u) + 0x00800000u;
    s = __uint_as_float(u);
  }
  return s;
}

// Round-to-nearest-even, saturating fp32 -> e4m3fn of two values; `lo` lands
// in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Correctly rounded fp32 quotient x / s of two pairs sharing one divisor,
// from r = RN(1/s) by Markstein's division correction (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with r within half an ulp of
// 1/s and q within one ulp of x/s, the residual e = x - q*s is exact under an
// FMA and RN(q + e*r) is the correctly rounded quotient.  The first estimate
// q0 = RN(x*r) can be up to two ulps off, so one correction step brings it
// within an ulp and a second one applies the theorem.  ns = -s.  Zeros keep
// their sign through a final copysign; quotients small enough to underflow
// fp32 all encode to a signed e4m3 zero, so the no-underflow premise does not
// matter for the codes.
__device__ __forceinline__ float2 quotient2(float2 x, float2 r, float2 ns) {
  float2 q = __fmul2_rn(x, r);
  q = __ffma2_rn(__ffma2_rn(q, ns, x), r, q);
  q = __ffma2_rn(__ffma2_rn(q, ns, x), r, q);
  q.x = __uint_as_float((__float_as_uint(q.x) & 0x7FFFFFFFu) | (__float_as_uint(x.x) & 0x80000000u));
  q.y = __uint_as_float((__float_as_uint(q.y) & 0x7FFFFFFFu) | (__float_as_uint(x.y) & 0x80000000u));
  return q;
}

// Quantizes 8 values of one block and packs the codes (element 0 in the low
// byte).  For ue8m0, r = 1/s is an exact power of two, so x * r is exactly
// the correctly rounded x / s; otherwise the quotient comes from quotient2.
// A block holding an infinity has s = inf and r = 0: the IEEE quotient of a
// finite x is then a signed zero, which the first estimate x * 0 already is,
// while the correction steps would compute 0 * inf = NaN.  With ns = 0 each
// step gives back its input (e = x, q + x * 0 = q), so the estimate stands.
template <bool UE8M0>
__device__ __forceinline__ uint2 quantize8(const float (&v)[8], float s, float r) {
  float t[8];
  if (UE8M0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = v[j] * r;
  } else {
    const float ns = isinf(s) ? 0.0f : -s;
    const float2 r2 = make_float2(r, r), ns2 = make_float2(ns, ns);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 q = quotient2(make_float2(v[2 * j], v[2 * j + 1]), r2, ns2);
      t[2 * j] = q.x;
      t[2 * j + 1] = q.y;
    }
  }
  uint2 out;
  out.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
  out.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
  return out;
}

// Self-test kernel: q[i] = x[i] / s[i] through quotient2.
__global__ void quotient_selftest_kernel(const float* __restrict__ x, const float* __restrict__ s,
                                         float* __restrict__ q, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    const float sc = s[i];
    const float2 r = make_float2(__frcp_rn(sc), 0.0f);
    q[i] = quotient2(make_float2(x[i], 0.0f), r, make_float2(-sc, -1.0f)).x;
  }
}

// s[i] = block_scale(amax[i]) for the self-test of the scale rule.
__global__ void scale_selftest_kernel(const float* __restrict__ amax, float* __restrict__ s,
                                      int64_t n, bool ue8m0) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * 256)
    s[i] = block_scale(amax[i], ue8m0);
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ---------------------------------------------------------------------------
// act_quant
// ---------------------------------------------------------------------------
// The input is a flat run of nblocks blocks of BLOCK elements (the last
// dimension is a multiple of BLOCK, so blocks never straddle rows) and block
// b's scale is s[b].  BLOCK / 32 lanes own one block, each holding 32
// consecutive elements; the amax is a log2(BLOCK / 32)-step xor shuffle among
// them, each thread computes the block's scale and writes its code bytes.  A
// warp covers 32 * 32 / BLOCK consecutive blocks per iteration with all loads
// issued first.  The pages' block size is 128 (the default of the
// block_size parameter); 32, 64 and 256 are the other sizes built.
constexpr int kActThreads = 256;
constexpr int kActUnroll = 1;
constexpr int kActElems = 32;

template <typename T, bool UE8M0, int BLOCK = 128>
__global__ void __launch_bounds__(kActThreads)
    act_quant_kernel(const T* __restrict__ x, uint8_t* __restrict__ q, float* __restrict__ s,
                     int64_t nblocks) {
  constexpr int kActLanes = BLOCK / kActElems;
  constexpr int kActBlocksPerWarp = 32 / kActLanes;
  static_assert(BLOCK == 32 || BLOCK == 64 || BLOCK == 128 || BLOCK == 256, "block size");
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int group = lane / kActLanes;
  const int li = lane % kActLanes;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kActThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kActThreads) >> 5;
  const int64_t step = nwarps * kActBlocksPerWarp * kActUnroll;

  for (int64_t base = warp * kActBlocksPerWarp * kActUnroll; base < nblocks; base += step) {
    float v[kActUnroll][kActElems];
#pragma unroll
    for (int u = 0; u < kActUnroll; ++u) {
      const int64_t b = base + kActBlocksPerWarp * u + group;
      if (b < nblocks) {
        const T* p = x + b * BLOCK + li * kActElems;
#pragma unroll
        for (int h = 0; h < kActElems / 8; ++h)
          load8(p + 8 * h, *reinterpret_cast<float(*)[8]>(&v[u][8 * h]));
      } else {
#pragma unroll
        for (int j = 0; j < kActElems; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kActUnroll; ++u) {
      const int64_t b = base + kActBlocksPerWarp * u + group;
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < kActElems; ++j) amax = fmaxf(amax, fabsf(v[u][j]));
#pragma unroll
      for (int off = kActLanes / 2; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
      const float sc = block_scale(amax, UE8M0);
      const float r = __frcp_rn(sc);
      if (b < nblocks) {
        uint8_t* qp = q + b * BLOCK + li * kActElems;
#pragma unroll
        for (int h = 0; h < kActElems / 16; ++h) {
          const uint2 lo = quantize8<UE8M0>(*reinterpret_cast<const float(*)[8]>(&v[u][16 * h]), sc, r);
          const uint2 hi =
              quantize8<UE8M0>(*reinterpret_cast<const float(*)[8]>(&v[u][16 * h + 8]), sc, r);
          __stcs(reinterpret_cast<uint4*>(qp + 16 * h), make_uint4(lo.x, lo.y, hi.x, hi.y));
        }
        if (li == 0) __stcs(s + b, sc);
      }
    }
  }
}

// Quotient n / d for a divisor fixed per launch, by multiplication
// (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", 1994, the round-up method): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, t = mulhi(m, n) and
// n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0).
struct InvariantDiv {
  uint32_t m, sh1, sh2;
};

// Multiplier and shifts for a divisor d >= 1 (host side, once per launch).
inline InvariantDiv invariant_div(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (uint64_t(1) << l) < d) ++l;
  const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1;
  return InvariantDiv{static_cast<uint32_t>(m), l < 1 ? l : 1u, l > 1 ? l - 1 : 0u};
}

__host__ __device__ __forceinline__ uint32_t div_invariant(uint32_t n, const InvariantDiv& d) {
#ifdef __CUDA_ARCH__
  const uint32_t t = __umulhi(n, d.m);
#else
  const uint32_t t = static_cast<uint32_t>((static_cast<uint64_t>(n) * d.m) >> 32);
#endif
  return (t + ((n - t) >> d.sh1)) >> d.sh2;
}

// ---------------------------------------------------------------------------
// act_quant with precomputed scales (the static activation scheme)
// ---------------------------------------------------------------------------
// Thread-chunks of kStaticElems consecutive elements of one row (it divides
// every block size, so a chunk has one scale): s[row * s_row_stride + (col >> lb)], with
// s_row_stride = 0 for per-channel-block scales shared by all rows.  With
// s_out, the chunk that starts a block also writes that scale to
// s_out[row, block] (the per-row table fp8_gemm reads).
//
// q = e4m3_satfinite(RN(x / s)).  For s in [2^-89, 2^100], r = RN(1/s) is a
// normal number and Markstein's correction (quotient2) yields the correctly
// rounded quotient whenever it is below 2^10 in magnitude and |x| >= 2^-100;
// below that |x / s| < 2^-11, which encodes to a signed zero whatever the
// rounding of the quotient.  A first estimate |x * r| >= 2^10 means a true
// quotient far above 448, which saturates: that estimate is used as it is
// (it may be infinite, and the correction would turn inf into NaN).  Scales
// outside that range (or not positive) take the IEEE division itself.
// 32 elements per thread and one chunk per loop step measured fastest on
// B200 (0.86 of the measured copy bandwidth on [16384, 7168] bf16; 16
// elements or two chunks per step held more registers and ran at 0.68-0.73).
constexpr int kStaticThreads = 256;
constexpr int kStaticUnroll = 1;
constexpr int kStaticElems = 32;   // elements per thread-chunk (divides every block size)

template <int E>
__device__ __forceinline__ void load_n(const __nv_bfloat16* p, float (&v)[E]) {
#pragma unroll
  for (int h = 0; h < E / 8; ++h) load8(p + 8 * h, *reinterpret_cast<float(*)[8]>(&v[8 * h]));
}
template <int E>
__device__ __forceinline__ void load_n(const float* p, float (&v)[E]) {
#pragma unroll
  for (int h = 0; h < E / 8; ++h) load8(p + 8 * h, *reinterpret_cast<float(*)[8]>(&v[8 * h]));
}

// Codes of 16 values sharing the scale sc (r = RN(1/sc) when `recip`).
__device__ __forceinline__ uint4 quantize16_given_scale(const float* v, float sc, float r,
                                                        bool recip) {
  float t[16];
  if (recip) {
    const float2 r2 = make_float2(r, r), ns2 = make_float2(-sc, -sc);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 x = make_float2(v[2 * j], v[2 * j + 1]);
      const float2 q0 = __fmul2_rn(x, r2);
      const float2 q = quotient2(x, r2, ns2);
      t[2 * j] = fabsf(q0.x) >= 1024.0f ? q0.x : q.x;
      t[2 * j + 1] = fabsf(q0.y) >= 1024.0f ? q0.y : q.y;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) t[j] = __fdiv_rn(v[j], sc);
  }
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    w[j] = e4m3x2(t[4 * j], t[4 * j + 1]) | (e4m3x2(t[4 * j + 2], t[4 * j + 3]) << 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T>
__global__ void __launch_bounds__(kStaticThreads)
    act_quant_static_kernel(const T* __restrict__ x, const float* __restrict__ s,
                            uint8_t* __restrict__ q, float* __restrict__ s_out,
                            uint32_t total_chunks, uint32_t chunks_per_row, InvariantDiv row_div,
                            int64_t s_row_stride, int64_t nblk, int lb) {
  pdl_trigger();
  pdl_wait();
  constexpr int E = kStaticElems;
  const uint32_t stride = gridDim.x * kStaticThreads * kStaticUnroll;
  for (uint32_t c0 = blockIdx.x * kStaticThreads * kStaticUnroll + threadIdx.x; c0 < total_chunks;
       c0 += stride) {
    float v[kStaticUnroll][E];
    float sc[kStaticUnroll];
#pragma unroll
    for (int u = 0; u < kStaticUnroll; ++u) {
      const uint32_t c = c0 + u * kStaticThreads;
      if (c < total_chunks) {
        const uint32_t row = div_invariant(c, row_div);
        const uint32_t col = (c - row * chunks_per_row) * E;
        load_n<E>(x + static_cast<int64_t>(c) * E, v[u]);
        sc[u] = __ldg(s + static_cast<int64_t>(row) * s_row_stride + (col >> lb));
      }
    }
#pragma unroll
    for (int u = 0; u < kStaticUnroll; ++u) {
      const uint32_t c = c0 + u * kStaticThreads;
      if (c >= total_chunks) continue;
      const bool recip = sc[u] >= 0x1p-89f && sc[u] <= 0x1p100f;
      const float r = recip ? __frcp_rn(sc[u]) : 0.0f;
      uint8_t* qp = q + static_cast<int64_t>(c) * E;
#pragma unroll
      for (int h = 0; h < E / 16; ++h)
        __stcs(reinterpret_cast<uint4*>(qp + 16 * h),
               quantize16_given_scale(&v[u][16 * h], sc[u], r, recip));
      if (s_out != nullptr) {
        const uint32_t row = div_invariant(c, row_div);
        const uint32_t col = (c - row * chunks_per_row) * E;
        if ((col & ((1u << lb) - 1u)) == 0)
          s_out[static_cast<int64_t>(row) * nblk + (col >> lb)] = sc[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// weight_dequant
// ---------------------------------------------------------------------------

// Value of an e4m3fn code, from the format definition: the 7 magnitude bits
// EEEE MMM placed at bit 20 of an fp32 pattern give an fp32 number whose
// exponent field is EEEE (bias 127 instead of 7) and whose fraction starts
// with MMM; multiplying by 2^120 restores the bias exactly, for subnormal
// codes too (they become fp32 subnormals, which are kept: no flush-to-zero).
// S.1111.111 is NaN.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t mag = code & 0x7Fu;
  float v = __uint_as_float(mag << 20) * 0x1p120f;
  v = (mag == 0x7Fu) ? __uint_as_float(0x7FC00000u) : v;
  return __uint_as_float(__float_as_uint(v) | ((code & 0x80u) << 24));
}

constexpr int kDeqThreads = 512;
constexpr int kDeqUnroll = 2;

// fp32 bits of (e4m3 value of the byte in bits 24..31 of c) * 2^-120: an
// arithmetic shift by 4 moves the 7 magnitude bits to 26..20 (exponent field
// e, mantissa m of e4m3 become the low exponent bits and top mantissa bits of
// fp32, which re-biases 7 -> 127) and the clear removes the sign's copies.
// Exact for normal and subnormal codes; the NaN codes are handled apart.
__device__ __forceinline__ float e4m3_times_2m120(uint32_t c_top) {
  return __uint_as_float(static_cast<uint32_t>(static_cast<int32_t>(c_top) >> 4) & 0x87FFFFFFu);
}

// Nonzero when one of the four code bytes of w is a NaN code (0x7F or 0xFF).
__device__ __forceinline__ uint32_t has_nan_code(uint32_t w) {
  return ((w & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u;
}

// Vector path (N % 16 == 0): a thread owns 16 consecutive codes of one row
// (one 16-byte load); all 16 share one scale because 16 divides every block
// size.  Chunk indices fit in 32 bits (the host checks M * N / 16 < 2^32).  Element
// (row, col) takes the scale s[(row >> row_shift) * s_row_stride + (col >> lb)]:
// row_shift = lb and s_row_stride = cdiv(N, block) for a weight's block x block
// tiles; row_shift = 0 for activations, s_row_stride = cols / block for a
// per-row table or 0 for static per-channel-block scales.  The fast
// path multiplies the shifted decode by s * 2^120, which is exact while
// |s| < 2^7 (the product of the real factors is q * s, rounded once, as in
// fl32(decode(q) * s)); chunks with a larger or non-finite scale, or with a
// NaN code, take the integer decode of e4m3_value.
template <bool OUT_BF16>
__global__ void __launch_bounds__(kDeqThreads)
    weight_dequant_kernel(const uint8_t* __restrict__ q, const float* __restrict__ s,
                          void* __restrict__ y, uint32_t total_chunks, uint32_t chunks_per_row,
                          InvariantDiv row_div, int64_t s_row_stride, int row_shift, int lb) {
  pdl_trigger();
  pdl_wait();
  const uint32_t stride = gridDim.x * kDeqThreads * kDeqUnroll;
  for (uint32_t c0 = blockIdx.x * kDeqThreads * kDeqUnroll + threadIdx.x; c0 < total_chunks;
       c0 += stride) {
    uint4 raw[kDeqUnroll];
    float sc[kDeqUnroll];
    int64_t off[kDeqUnroll];
#pragma unroll
    for (int u = 0; u < kDeqUnroll; ++u) {
      const uint32_t c = c0 + u * kDeqThreads;
      if (c < total_chunks) {
        const uint32_t row = div_invariant(c, row_div);
        const uint32_t col = (c - row * chunks_per_row) * 16;
        off[u] = static_cast<int64_t>(c) * 16;
        raw[u] = __ldcs(reinterpret_cast<const uint4*>(q + off[u]));
        sc[u] = __ldg(s + static_cast<int64_t>(row >> row_shift) * s_row_stride + (col >> lb));
      } else {
        off[u] = -1;
      }
    }
#pragma unroll
    for (int u = 0; u < kDeqUnroll; ++u) {
      if (off[u] < 0) continue;
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      float v[16];
      const bool fast = fabsf(sc[u]) < 128.0f &&
                        (has_nan_code(w[0]) | has_nan_code(w[1]) | has_nan_code(w[2]) |
                         has_nan_code(w[3])) == 0u;
      if (fast) {
        const float sc_up = sc[u] * 0x1p120f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[4 * j + 0] = e4m3_times_2m120(w[j] << 24) * sc_up;
          v[4 * j + 1] = e4m3_times_2m120(__byte_perm(w[j], 0u, 0x1444u)) * sc_up;
          v[4 * j + 2] = e4m3_times_2m120(__byte_perm(w[j], 0u, 0x2444u)) * sc_up;
          v[4 * j + 3] = e4m3_times_2m120(w[j] & 0xFF000000u) * sc_up;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = e4m3_value((w[j >> 2] >> (8 * (j & 3))) & 0xFFu) * sc[u];
      }
      if (OUT_BF16) {
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
          h[j] = *reinterpret_cast<uint32_t*>(&b2);
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + off[u]);
        __stcs(dst, make_uint4(h[0], h[1], h[2], h[3]));
        __stcs(dst + 1, make_uint4(h[4], h[5], h[6], h[7]));
      } else {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + off[u]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          __stcs(dst + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
      }
    }
  }
}

// Element path for any N (ragged widths that are not a multiple of 16).
template <bool OUT_BF16>
__global__ void __launch_bounds__(kDeqThreads)
    weight_dequant_any_kernel(const uint8_t* __restrict__ q, const float* __restrict__ s,
                              void* __restrict__ y, int64_t M, int64_t N, int64_t s_row_stride,
                              int row_shift, int lb) {
  pdl_trigger();
  pdl_wait();
  const int64_t total = M * N;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDeqThreads + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kDeqThreads) {
    const int64_t row = i / N, col = i - row * N;
    const float v = e4m3_value(q[i]) * __ldg(s + (row >> row_shift) * s_row_stride + (col >> lb));
    if (OUT_BF16)
      static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(y)[i] = v;
  }
}

// ---------------------------------------------------------------------------
// weight_quant: one CTA per block x block tile (partial at the edges)
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename T>
__global__ void __launch_bounds__(256)
    weight_quant_kernel(const T* __restrict__ w, uint8_t* __restrict__ q, float* __restrict__ s,
                        int64_t M, int64_t N, int64_t nbn, bool ue8m0, int lb) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const int64_t bi = blockIdx.y, bj = blockIdx.x;
  const int blk = 1 << lb;
  const int64_t r0 = bi * blk, c0 = bj * blk;
  const int rows = static_cast<int>(M - r0 < blk ? M - r0 : blk);
  const int cols = static_cast<int>(N - c0 < blk ? N - c0 : blk);
  float amax = 0.0f;
  for (int e = threadIdx.x; e < (rows << lb); e += 256) {
    const int r = e >> lb, c = e & (blk - 1);
    if (c < cols) amax = fmaxf(amax, fabsf(load_elem(w + (r0 + r) * N + c0 + c)));
  }
  for (int off = 16; off >= 1; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = block_scale(amax, ue8m0);
  if (threadIdx.x == 0) s[bi * nbn + bj] = sc;
  for (int e = threadIdx.x; e < (rows << lb); e += 256) {
    const int r = e >> lb, c = e & (blk - 1);
    if (c < cols) {
      const int64_t i = (r0 + r) * N + c0 + c;
      q[i] = static_cast<uint8_t>(e4m3x2(__fdiv_rn(load_elem(w + i), sc), 0.0f) & 0xFFu);
    }
  }
}

// weight_quant for 128 x 128 tiles, one pass: the tile stays in registers.
// Thread t owns columns 4 * (t % 32) .. +3 of rows t / 32 + 8 k (k < 16), so
// every warp-wide load reads 128 consecutive elements of one row and every
// warp-wide store writes 128 consecutive codes.  The tile amax is a warp
// shuffle then a reduction over the 8 warps in shared memory; the scale is the
// act_quant rule and each quotient is the correctly rounded w / s (Markstein's
// correction, as in act_quant), so the codes are those of the two-pass
// kernel.  Elements past the matrix's ragged edges read as 0 and are not
// stored.
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 raw = __ldcs(reinterpret_cast<const uint2*>(p));
  v[0] = __uint_as_float(raw.x << 16);
  v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  v[2] = __uint_as_float(raw.y << 16);
  v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
}

template <typename T>
__global__ void __launch_bounds__(256)
    weight_quant128_kernel(const T* __restrict__ w, uint8_t* __restrict__ q, float* __restrict__ s,
                           int64_t M, int64_t N, int64_t nbn, bool ue8m0, bool vec_ok) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 128, c0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int64_t col = c0 + 4 * lane;
  float v[16][4];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int64_t row = r0 + wid + 8 * k;
    if (row < M && vec_ok && col + 4 <= N) {
      load4(w + row * N + col, v[k]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[k][j] = (row < M && col + j < N) ? load_elem(w + row * N + col + j) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fabsf(v[k][j]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if (lane == 0) red[wid] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = block_scale(amax, ue8m0);
  if (threadIdx.x == 0) s[static_cast<int64_t>(blockIdx.y) * nbn + blockIdx.x] = sc;
  const float r = __frcp_rn(sc);
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    const float v8[8] = {v[k][0], v[k][1], v[k][2], v[k][3], v[k + 1][0], v[k + 1][1], v[k + 1][2], v[k + 1][3]};
    const uint2 c = ue8m0 ? quantize8<true>(v8, sc, r) : quantize8<false>(v8, sc, r);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t row = r0 + wid + 8 * (k + h);
      const uint32_t codes = h ? c.y : c.x;
      if (row >= M) continue;
      if (vec_ok && col + 4 <= N) {
        *reinterpret_cast<uint32_t*>(q + row * N + col) = codes;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col + j < N) q[row * N + col + j] = static_cast<uint8_t>(codes >> (8 * j));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Split-K reduction: y[m, n] = sum_s ws[s][m][n], summed in split order, as
// bf16 (rounded to nearest even) or FP32.
// ---------------------------------------------------------------------------
template <typename OutT>
__global__ void __launch_bounds__(256)
    splitk_reduce_kernel(const float* __restrict__ ws, OutT* __restrict__ y,
                         int64_t MN, int splits) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < MN;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    float acc = 0.0f;
    for (int sp = 0; sp < splits; ++sp) acc += ws[sp * MN + i];
    if constexpr (std::is_same_v<OutT, float>)
      y[i] = acc;
    else
      y[i] = __float2bfloat16_rn(acc);
  }
}

}  // namespace fp8bs
