// The FP8 linear layer with act_quant inside the GEMM launch ("Understanding
// Dynamic and Static Activation Quantization Schemes in DeepSeek-V3", section
// "How Dynamic Activation Quantization Works": the linear layer quantizes its
// input with act_quant during the forward pass, then runs fp8_gemm).
//
// When the GEMM's output tiles fill only part of the GPU (a narrow N such as
// 576), the launch gives the idle SMs to the quantization.  CTAs below
// gemm_ctas run the GEMM as fp8_gemm_kernel always does; the others are
// quantizer CTAs.  A quantizer CTA streams 128-row x 128-column chunks of x
// (one K block of one m tile) into a ring of shared-memory stages by TMA,
// computes exactly what act_quant computes for each 1 x 128 block (amax,
// block_scale, the correctly rounded quotient, the saturating e4m3 cast),
// writes the codes and scales to the caller's q and s, and then counts
// itself into the chunk's ready flag (release at GPU scope).  Chunks go K-block-major, the
// order in which the GEMM's tiles consume them, so the GEMM runs a few K
// blocks behind the quantization instead of after all of it.  A GEMM CTA's
// TMA producer and scale producer wait for a chunk's flag (acquire) before
// they read its codes or scales.  Nothing is quantized twice: every chunk
// has one quantizer.
#pragma once

#include "quant.cuh"
#include "sm100.cuh"

namespace fp8bs {
namespace gemm {

constexpr int kQBoxBytes = 128 * 64 * 2;        // 128 rows x 64 bf16 columns (128-byte swizzle)
constexpr int kQChunkBytes = 2 * kQBoxBytes;    // one (m tile, K block) chunk of x
constexpr int kQStages = 6;
constexpr int kQWarps = 8;                      // quantizing warps 1 .. kQWarps
constexpr int kQRingBytes = kQStages * kQChunkBytes;
constexpr int kQBarBytes = 256;

// Waits until all kQWarps quantizer warps have counted themselves into the
// chunk flag *f, acquiring their writes.
// Bounded like the mbarrier waits: after kWaitLimitNs it records
// FP8BS_ERR_TIMEOUT, raises *abort and returns false.
__device__ __forceinline__ bool wait_chunk_flag(const int* f, volatile int* abort) {
  auto ready = [&]() {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v >= kQWarps;
  };
  if (ready()) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      if (ready()) return true;
      __nanosleep(64);
    }
    if (abort != nullptr && *abort) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      report_error(5);
      if (abort != nullptr) *abort = 1;
      return false;
    }
  }
}

// Orders the generic-proxy reads before it (the flag) with the tensor-copy
// (async proxy) reads of global memory after it.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// A quantizer CTA: qi-th of nq.  x is read through tmap_x (bf16 [M, K],
// boxes of 128 rows x 64 columns, 128-byte swizzle); q [M, K] e4m3 codes and
// s [M, K / 128] scales are written for rows below M; flags [m_tiles][kbn].
// Warp 0 lane 0 loads, warps 1 .. kQWarps quantize (16 rows each: four lanes
// per row, 32 columns per lane, two 8-row steps), free each stage and count
// each chunk in a shared-memory counter per warp; warp kQWarps + 1 lane 0
// announces, in chunk order, every chunk all warps have counted, by a
// release at GPU scope per chunk flag.  A fence per chunk in the quantizing
// warps themselves would stall each of them for the round trip of its own
// stores.
template <bool UE8M0>
__device__ __forceinline__ void quantize_cta(const CUtensorMap* tmap_x, int64_t M, int K,
                                             uint8_t* __restrict__ q, float* __restrict__ s,
                                             int* __restrict__ flags, uint8_t* smem, int qi,
                                             int nq) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQRingBytes);
  uint64_t* empty = full + kQStages;
  // done[w]: chunks quantizing warp w has finished (its stores issued).
  uint32_t* done = reinterpret_cast<uint32_t*>(empty + kQStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(done + kQWarps);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kbn = K / 128;
  const int m_tiles = static_cast<int>((M + 127) / 128);
  const int chunks = m_tiles * kbn;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kQStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kQWarps);
    }
    for (int w = 0; w < kQWarps; ++w) done[w] = 0;
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_descriptor(tmap_x);
      uint32_t i = 0, armed = 0, armed_phase = 0;
      for (int c = qi; c < chunks; c += nq, ++i) {
        const int st = static_cast<int>(i % kQStages);
        const uint32_t ph = (i / kQStages) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) break;
        const int kb = c / m_tiles, m = c - kb * m_tiles;
        mbar_arrive_expect_tx(&full[st], kQChunkBytes);
        uint8_t* dst = smem + st * kQChunkBytes;
        tma_load_2d(dst, tmap_x, &full[st], kb * 128, m * 128);
        tma_load_2d(dst + kQBoxBytes, tmap_x, &full[st], kb * 128 + 64, m * 128);
        armed |= 1u << st;
        armed_phase = (armed_phase & ~(1u << st)) | (ph << st);
      }
      if (*abort_flag) {
        // Let every load in flight land before the CTA exits.
        for (int st = 0; st < kQStages; ++st)
          if (armed & (1u << st)) mbar_wait(&full[st], (armed_phase >> st) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp <= kQWarps) {
    // Four lanes per 128-column row, 32 columns (four 16-byte units) each, as
    // in act_quant: lane 4 g + t takes row (warp step) * 8 + g, columns
    // 32 t .. 32 t + 31, which lie in box t / 2, units 4 (t % 2) .. + 3.
    const int cw = warp - 1;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int hb = t >> 1;
    const int u0 = (t & 1) * 4;
    uint32_t i = 0;
    for (int c = qi; c < chunks; c += nq, ++i) {
      const int st = static_cast<int>(i % kQStages);
      const uint32_t ph = (i / kQStages) & 1u;
      const bool ok = mbar_wait(&full[st], ph, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const int kb = c / m_tiles, m = c - kb * m_tiles;
      const uint8_t* box = smem + st * kQChunkBytes + hb * kQBoxBytes;
      // This warp's two 8-row steps of the chunk, side by side so that their
      // dependency chains overlap.
      constexpr int R = 2;
      float v[R][32];
      float amax[R];
      int rr[R];
#pragma unroll
      for (int k = 0; k < R; ++k) {
        rr[k] = (cw * R + k) * 8 + g;
        amax[k] = 0.0f;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          // 128-byte swizzle: unit u of box row r sits at unit u ^ (r % 8).
          const uint4 raw = *reinterpret_cast<const uint4*>(
              box + rr[k] * 128 + (((u0 + uu) ^ (rr[k] & 7)) << 4));
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[k][8 * uu + 2 * e] = __uint_as_float(w[e] << 16);
            v[k][8 * uu + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            amax[k] = fmaxf(amax[k], fmaxf(fabsf(v[k][8 * uu + 2 * e]),
                                           fabsf(v[k][8 * uu + 2 * e + 1])));
          }
        }
      }
#pragma unroll
      for (int off = 2; off >= 1; off >>= 1)
#pragma unroll
        for (int k = 0; k < R; ++k) amax[k] = fmaxf(amax[k], __shfl_xor_sync(0xFFFFFFFFu, amax[k], off));
      float sc[R], rc[R];
#pragma unroll
      for (int k = 0; k < R; ++k) {
        sc[k] = block_scale(amax[k], UE8M0);
        rc[k] = __frcp_rn(sc[k]);
      }
#pragma unroll
      for (int k = 0; k < R; ++k) {
        uint32_t codes[8];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const uint2 cc = quantize8<UE8M0>(*reinterpret_cast<const float(*)[8]>(&v[k][8 * hh]),
                                            sc[k], rc[k]);
          codes[2 * hh] = cc.x;
          codes[2 * hh + 1] = cc.y;
        }
        const int64_t row = static_cast<int64_t>(m) * 128 + rr[k];
        if (row < M) {
          uint4* dst = reinterpret_cast<uint4*>(q + row * K + kb * 128 + t * 32);
          dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
          dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
          if (t == 0) s[row * kbn + kb] = sc[k];
        }
      }
      // This warp is done with the chunk: it has read the stage, and its
      // count (a release at CTA scope) hands its stores to the announcer.
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[st]);
        asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_addr(done + cw)),
                     "r"(i + 1)
                     : "memory");
      }
    }
  } else if (warp == kQWarps + 1) {
    if (lane == 0) {
      // Chunks in order: once every quantizing warp has counted past chunk i,
      // its flag is published by a release at GPU scope, which carries the
      // warps' stores acquired through their counts (cumulativity).
      uint32_t i = 0;
      const uint64_t t_limit = kWaitLimitNs;
      uint64_t t0 = global_timer_ns();
      for (int c = qi; c < chunks;) {
        uint32_t least = 0xFFFFFFFFu;
#pragma unroll
        for (int w = 0; w < kQWarps; ++w) {
          uint32_t d;
          asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(d) : "r"(smem_addr(done + w))
                       : "memory");
          least = d < least ? d : least;
        }
        if (least <= i) {
          if (*abort_flag) break;
          if (global_timer_ns() - t0 > t_limit) {
            report_error(5);
            *abort_flag = 1;
            break;
          }
          __nanosleep(32);
          continue;
        }
        for (; i < least && c < chunks; ++i, c += nq) {
          const int kb = c / m_tiles, m = c - kb * m_tiles;
          asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(flags + m * kbn + kb),
                       "r"(kQWarps)
                       : "memory");
        }
        t0 = global_timer_ns();
      }
    }
    __syncwarp();
  }
  __syncthreads();
}

}  // namespace gemm
}  // namespace fp8bs
