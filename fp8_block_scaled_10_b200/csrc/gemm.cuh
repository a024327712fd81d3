// Block-scaled FP8 GEMM for sm_100a: y = A * W^T with A [M, K] and W [N, K]
// in e4m3fn, activation scales a_s [M, K/128] (one per 1x128 block) and weight
// scales w_s [cdiv(N,128), K/128] (one per 128x128 block), FP32 accumulation,
// bf16 output:
//   y[m, n] = sum_kb a_s[m, kb] * w_s[n/128, kb] * P_kb[m, n],
//   P_kb    = sum over the 128 k of block kb of A[m, k] * W[n, k].
// ("How weight_dequant Handles Per-Block Scaling in DeepSeek-V3 FP8 GEMM",
// section "Relationship to FP8 GEMM Operations": fp8_gemm(a, a_s, b, b_s) with
// the scaling fused into the matrix product; "DeepSeek-V3: How Selective FP8
// Stays Stable", section "Learning outcomes": partial sums promoted to FP32.)
//
// Blackwell form of the promotion.  Each 128-wide K block is one group of four
// tcgen05.mma (K = 32 each) that writes a fresh FP32 partial P_kb into one of
// two TMEM buffers; the epilogue warps read it back with tcgen05.ld and fold
// it into register accumulators with one FMA per element by
// a_s[m, kb] * w_s[nb, kb], while the tensor core fills the other buffer.
//
// Roles (persistent CTAs, one per SM, walking work units in a fixed order):
//   warp 0     TMA producer: A tile [128 x 128] and W tile into a ring of
//              shared-memory stages (128B swizzle).
//   warp 1     owns the TMEM allocation; one lane issues the MMAs.
//   epilogue   8 warps from kFirstEpiWarp: warp w reads TMEM lanes
//              32*(w%4)..+31 (one output row per thread) and BN/2 columns
//              (column half (w - kFirstEpiWarp) / 4).  Loads of the next
//              32-column chunk overlap the FMAs of the current one.
// Pair mode (PAIR): two CTAs of a cluster share one tcgen05.mma.cta_group::2
// of M = 256.  Each CTA loads its own 128 rows of A and its own half of the W
// tile (BN/2 rows), so each SM moves a third less operand data per MMA than
// a single CTA with a 128 x BN tile.  The leader (even) CTA issues the MMAs;
// both CTAs' loads complete on the leader's full barrier, the leader's commits
// arrive on both CTAs' barriers, and both CTAs' epilogues release the TMEM
// buffer on the leader's barrier.  Each CTA holds its own 128 rows of the
// accumulator in its own TMEM.
//
// A work unit is (m tile, n tile, K split).  With one split the epilogue
// writes bf16; with several it writes FP32 partials that a reduction kernel
// sums.  Grouped mode (experts) walks (expert, m tile, n tile) units whose
// rows come from device-side prefix offsets.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace fp8bs {
namespace gemm {

constexpr int BM = 128;      // rows of A per CTA
constexpr int BK = 128;      // one K block per pipeline stage
constexpr int kMaxGroups = 1024;

struct Params {
  const float* sa;          // [M_total, kbn]
  const float* sw;          // [G][nbn][kbn]
  __nv_bfloat16* y;         // [M_total, N]
  float* ws;                // [splits][M][N] FP32 partials when splits > 1
  const int64_t* m_offsets; // grouped mode: [G + 1] prefix row offsets (device)
  int64_t M;                // rows of A (M_total in grouped mode)
  int N;
  int kbn;                  // K / 128
  int nbn;                  // cdiv(N, 128)
  int m_tiles;              // dense mode: tiles of kUnitRows rows
  int n_tiles;
  int splits;
  int kb_per_split;
  int num_units;            // dense mode; grouped mode derives it on the device
  int groups;               // grouped mode
  int y_tma;                // 1: bf16 y written by TMA stores through staging boxes;
                            // 2: FP32 split-K partials written by TMA stores (3-D map)
};

// Output staging for TMA stores of bf16 y: each epilogue warp owns one box of
// 32 rows x 32 columns (2 KB) in shared memory, laid out in the 64-byte
// swizzle of the y tensor map (16-byte chunk q of row r at chunk
// q ^ ((r >> 1) & 3)), so the 32 lanes writing one row each hit distinct
// banks.  One TMA store then writes 32 rows x 64 B of y; the warps' direct
// stores would write 16 B into 32 different rows per instruction.
constexpr int kOutBoxBytes = 32 * 32 * 2;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b2);
}

// Stages this lane's 64 bytes (32 packed bf16, or 16 FP32 split-K partials)
// as row `lane` of the warp's box and stores the box at column x, row y of y
// (2-D map), or of split z of the FP32 workspace (3-D map, z >= 0).  Lane 0
// first waits until the box's previous store has read it.
__device__ __forceinline__ void store_out_box(const CUtensorMap* tmap, uint8_t* box, int lane,
                                              const uint32_t (&h)[16], int32_t x, int32_t y,
                                              int32_t z = -1) {
  if (lane == 0) tma_store_wait_read();
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(box + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (z < 0) tma_store_2d(tmap, box, x, y);
    else tma_store_3d(tmap, box, x, y, z);
    tma_store_commit();
  }
}

template <int BN, bool PAIR>
struct Cfg {
  static constexpr int kUnitRows = PAIR ? 2 * BM : BM;   // rows of one work unit
  static constexpr int kBRows = PAIR ? BN / 2 : BN;      // W rows loaded per CTA
  static constexpr int kABytes = BM * BK;
  static constexpr int kBBytes = kBRows * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (6 * 32768) / kStageBytes;
  // Two epilogue warpgroups: each covers all 128 TMEM lanes (one warp per
  // 32-lane quadrant) and half of the tile's columns.
  static constexpr int kEpiWarps = 8;
  static constexpr int kColsPerWarp = BN / 2;
  static constexpr int kChunks = kColsPerWarp / 32;
  // BN = 256: warps 0-3 form a control warpgroup that hands registers to the
  // two epilogue warpgroups (setmaxnreg); BN = 128: warps 0-1 control, 2-9
  // epilogue, and every thread can hold its 64 accumulators at launch.
  static constexpr int kFirstEpiWarp = (BN == 256) ? 4 : 2;
  static constexpr bool kSplitRegs = (BN == 256);
  static constexpr int kCtrlRegs = 56;
  static constexpr int kEpiRegs = 224;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr int kTmemCols = 2 * BN;
  // In pair mode with BN = 256 each K block's MMA is issued as two sub-MMAs of
  // N = 128, each into its own TMEM sub-buffer with its own full/empty
  // barrier pair, so the epilogue warps of column half g can drain sub-buffer
  // g while the tensor core still works on the other half; each sub-MMA takes
  // 64 rows of W from each CTA, so a CTA loads two chunks of 64 rows per
  // stage.  (A single CTA keeps one N = BN MMA: two N = 128 MMAs would read
  // the A tile from shared memory twice.)
  static constexpr int kSplitN = (PAIR && BN == 256) ? 2 : 1;
  static constexpr int kSubN = BN / kSplitN;
  static constexpr int kBChunkRows = PAIR ? kSubN / 2 : kSubN;
  static constexpr int kBChunkBytes = kBChunkRows * BK;
  static constexpr int kSubBuffers = 2 * kSplitN;
  static constexpr int kCtrlBytes = 256;
  // grouped mode: per-group m-tile prefix (int)
  static constexpr int kGroupBytes = 4 * (kMaxGroups + 1);
  // output staging boxes (one per epilogue warp), 1024-byte aligned
  __host__ __device__ static constexpr int out_offset(bool grouped) {
    return (kStages * kStageBytes + kCtrlBytes + (grouped ? kGroupBytes : 0) + 1023) & ~1023;
  }
  __host__ __device__ static constexpr int smem_bytes(bool grouped) {
    return out_offset(grouped) + kEpiWarps * kOutBoxBytes + 1024;
  }
  // Arrivals that release one TMEM sub-buffer: the epilogue warps that read
  // it, in both CTAs in pair mode.
  static constexpr int kTmemReleaseCount = (kEpiWarps / kSplitN) * (PAIR ? 2 : 1);
};

// Control block at the end of the tile ring.
template <int kStages>
struct Ctrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[4];     // [buffer * kSplitN + half]
  uint64_t tempty[4];
  uint64_t flush;
  uint32_t tmem_base;
  int abort_flag;
  int num_units;
};

struct Unit {
  int64_t row0;      // first A/y row of the unit (of the pair in pair mode)
  int64_t row_end;   // rows >= row_end are not stored
  int64_t w_row0;    // first W row (grouped: expert * N + n0)
  int group;
  int n_tile;
  int kb0, kb1;
  int split;
};

// Dense units: m tile fastest, so the CTAs running at the same time share W
// tiles (and sweep all of A, which stays in L2).
template <int kUnitRows>
__device__ __forceinline__ Unit dense_unit(const Params& p, int u) {
  Unit t;
  const int m_tile = u % p.m_tiles;
  const int rest = u / p.m_tiles;
  t.split = rest % p.splits;
  t.n_tile = rest / p.splits;
  t.group = 0;
  t.row0 = static_cast<int64_t>(m_tile) * kUnitRows;
  t.row_end = p.M;
  t.kb0 = t.split * p.kb_per_split;
  t.kb1 = min(p.kbn, t.kb0 + p.kb_per_split);
  return t;
}

// Row range [lo, hi) of group g: the device offsets clamped to [0, M] and
// made non-decreasing.
__device__ __forceinline__ void group_rows(const Params& p, int g, int64_t& lo, int64_t& hi) {
  lo = __ldg(p.m_offsets + g);
  hi = __ldg(p.m_offsets + g + 1);
  lo = lo < 0 ? 0 : (lo > p.M ? p.M : lo);
  hi = hi < lo ? lo : (hi > p.M ? p.M : hi);
}

// Grouped units: n tile fastest inside one global m tile, so the CTAs running
// at the same time work on one or two experts and read each W_e once.
// tile_prefix[g] is the number of m tiles of groups < g.
template <int kUnitRows>
__device__ __forceinline__ Unit grouped_unit(const Params& p, const int* tile_prefix, int u) {
  Unit t;
  const int gm = u / p.n_tiles;
  t.n_tile = u % p.n_tiles;
  int a = 0, b = p.groups;
  while (b - a > 1) {
    const int mid = (a + b) >> 1;
    if (tile_prefix[mid] <= gm) a = mid; else b = mid;
  }
  t.group = a;
  int64_t lo, hi;
  group_rows(p, a, lo, hi);
  t.row0 = lo + static_cast<int64_t>(gm - tile_prefix[a]) * kUnitRows;
  t.row_end = hi;
  t.split = 0;
  t.kb0 = 0;
  t.kb1 = p.kbn;
  return t;
}

template <int BN, bool GROUPED, bool PAIR>
__global__ void __launch_bounds__(Cfg<BN, PAIR>::kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  using C = Cfg<BN, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + C::kStages * C::kABytes;
  Ctrl<C::kStages>* ctrl = reinterpret_cast<Ctrl<C::kStages>*>(smem + C::kStages * C::kStageBytes);
  static_assert(sizeof(Ctrl<C::kStages>) <= C::kCtrlBytes, "control block too large");
  uint64_t* full = ctrl->full;
  uint64_t* empty = ctrl->empty;
  uint64_t* tfull = ctrl->tfull;
  uint64_t* tempty = ctrl->tempty;
  uint64_t* flush = &ctrl->flush;
  volatile int* abort_flag = &ctrl->abort_flag;
  int* tile_prefix = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes + C::kCtrlBytes);
  uint8_t* out_boxes = smem + C::out_offset(GROUPED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  const uint32_t rank = PAIR ? cluster_rank() : 0u;   // 0 = leader
  const int unit_start = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int unit_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kSubBuffers; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kTmemReleaseCount);
    }
    mbar_init(flush, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_descriptor(&tmap_a);
    tma_prefetch_descriptor(&tmap_w);
    if (p.y_tma) tma_prefetch_descriptor(&tmap_y);
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(&ctrl->tmem_base, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&ctrl->tmem_base, C::kTmemCols);
      tmem_relinquish();
    }
  }
  // Inputs may come from the previous kernel of the stream (launched with
  // programmatic serialization): wait for it before any global access.
  pdl_wait();
  if (GROUPED) {
    // Clamp the device offsets to [0, M], count each group's m tiles and form
    // their exclusive prefix sum (warp 2, 32 groups per step).
    if (warp == 2) {
      int carry = 0;
      for (int g0 = 0; g0 < p.groups; g0 += 32) {
        const int g = g0 + lane;
        int tiles = 0;
        if (g < p.groups) {
          int64_t lo, hi;
          group_rows(p, g, lo, hi);
          tiles = static_cast<int>((hi - lo + C::kUnitRows - 1) / C::kUnitRows);
        }
        int incl = tiles;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
          if (lane >= off) incl += v;
        }
        if (g < p.groups) tile_prefix[g] = carry + incl - tiles;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (lane == 0) {
        tile_prefix[p.groups] = carry;
        ctrl->num_units = carry * p.n_tiles;
      }
    }
  } else if (threadIdx.x == 0) {
    ctrl->num_units = p.num_units;
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctrl->tmem_base;
  const int num_units = ctrl->num_units;

  auto unit_of = [&](int u) -> Unit {
    Unit t;
    if (GROUPED) {
      t = grouped_unit<C::kUnitRows>(p, tile_prefix, u);
      t.w_row0 = static_cast<int64_t>(t.group) * p.N + static_cast<int64_t>(t.n_tile) * BN;
    } else {
      t = dense_unit<C::kUnitRows>(p, u);
      t.w_row0 = static_cast<int64_t>(t.n_tile) * BN;
    }
    return t;
  };

  if (warp < C::kFirstEpiWarp) {
    if (C::kSplitRegs) reg_release<C::kCtrlRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;       // stages with a TMA load issued
      uint32_t armed_phase = 0; // parity each armed stage completes
      for (int u = unit_start; u < num_units; u += unit_step) {
        const Unit t = unit_of(u);
        const int32_t a_row = static_cast<int32_t>(t.row0 + rank * BM);
        // W rows of chunk h: sub-tile h (kSubN rows) and, in pair mode, this
        // CTA's half of it.
        const int32_t b_row = static_cast<int32_t>(t.w_row0 + rank * C::kBChunkRows);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
          if (PAIR) {
            // Both CTAs' bytes complete on the leader's full barrier, which the
            // leader alone arms.
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
            const uint32_t bar = map_to_rank(&full[stage], 0);
            tma_load_2d_pair(a_tiles + stage * C::kABytes, &tmap_a, bar, kb * BK, a_row);
#pragma unroll
            for (int h = 0; h < C::kSplitN; ++h)
              tma_load_2d_pair(b_tiles + stage * C::kBBytes + h * C::kBChunkBytes, &tmap_w, bar,
                               kb * BK, b_row + h * C::kSubN);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
            tma_load_2d(a_tiles + stage * C::kABytes, &tmap_a, &full[stage], kb * BK, a_row);
#pragma unroll
            for (int h = 0; h < C::kSplitN; ++h)
              tma_load_2d(b_tiles + stage * C::kBBytes + h * C::kBChunkBytes, &tmap_w,
                          &full[stage], kb * BK, b_row + h * C::kSubN);
          }
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (*abort_flag && (!PAIR || rank == 0)) {
        // Let every load in flight land before the CTA exits (in pair mode the
        // leader's full barriers count the peer's loads too).
        for (int s = 0; s < C::kStages; ++s)
          if (armed & (1u << s)) mbar_wait<PAIR>(&full[s], (armed_phase >> s) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && (!PAIR || rank == 0)) {
      constexpr uint32_t idesc = idesc_e4m3_f32(PAIR ? 2 * BM : BM, C::kSubN);
      int stage = 0;
      uint32_t phase = 0;
      int tb = 0;
      uint32_t tphase = 0;
      for (int u = unit_start; u < num_units; u += unit_step) {
        const Unit t = unit_of(u);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait<PAIR>(&full[stage], phase, abort_flag)) goto mma_done;
          tc_fence_after();
          const uint32_t a_addr = smem_addr(a_tiles + stage * C::kABytes);
          const uint32_t b_addr = smem_addr(b_tiles + stage * C::kBBytes);
#pragma unroll
          for (int h = 0; h < C::kSplitN; ++h) {
            const int sb = tb * C::kSplitN + h;
            if (!mbar_wait<PAIR>(&tempty[sb], tphase ^ 1u, abort_flag)) goto mma_done;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * BN + h * C::kSubN);
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
              const uint64_t ad = smem_desc_k_sw128(a_addr + 32 * k);
              const uint64_t bd = smem_desc_k_sw128(b_addr + h * C::kBChunkBytes + 32 * k);
              if (PAIR) mma_f8f6f4_pair(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
              else mma_f8f6f4(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
            }
            if (PAIR) mma_commit_pair_mask(&tfull[sb], 0x3);
            else mma_commit(&tfull[sb]);
          }
          if (PAIR) mma_commit_pair_mask(&empty[stage], 0x3);
          else mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
          tb ^= 1;
          if (tb == 0) tphase ^= 1u;
        }
      }
    mma_done:
      // Every MMA issued must finish before the TMEM columns are released.
      if (PAIR) mma_commit_pair(flush); else mma_commit(flush);
      mbar_wait(flush, 0, nullptr);
    }
    __syncwarp();
  }
  } else {
    if (C::kSplitRegs) reg_acquire<C::kEpiRegs>();
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::kFirstEpiWarp;
    const int quad = warp & 3;
    const int g = e >> 2;                       // column half
    constexpr int CPW = C::kColsPerWarp;
    constexpr int NCH = C::kChunks;
    const int row_in_tile = static_cast<int>(rank) * BM + quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const bool vec_store = (p.N % 8) == 0;
    // This warp's sub-buffer within each TMEM buffer (both halves are the same
    // sub-buffer when the MMA is not split).
    const int half = (g * C::kSplitN) >> 1;
    const uint32_t tempty_leader0 = PAIR ? map_to_rank(&tempty[half], 0) : 0u;
    const uint32_t tempty_leader1 = PAIR ? map_to_rank(&tempty[C::kSplitN + half], 0) : 0u;
    int tb = 0;
    uint32_t tphase = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      const int64_t row = t.row0 + row_in_tile;
      const bool row_ok = row < t.row_end;
      const int nb = (t.n_tile * BN + g * CPW) / 128;
      const bool nb_ok = nb < p.nbn;
      const float* sa_row = p.sa + (row_ok ? row : 0) * static_cast<int64_t>(p.kbn);
      const float* sw_row =
          p.sw + (static_cast<int64_t>(t.group) * p.nbn + (nb_ok ? nb : 0)) * p.kbn;
      float2 acc[CPW / 2];
#pragma unroll
      for (int j = 0; j < CPW / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
      float sa_next = row_ok ? __ldg(sa_row + t.kb0) : 0.0f;
      float sw_next = nb_ok ? __ldg(sw_row + t.kb0) : 0.0f;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const float scale = sa_next * sw_next;
        const float2 scale2 = make_float2(scale, scale);
        if (kb + 1 < t.kb1) {
          sa_next = row_ok ? __ldg(sa_row + kb + 1) : 0.0f;
          sw_next = nb_ok ? __ldg(sw_row + kb + 1) : 0.0f;
        }
        const bool ok = mbar_wait<PAIR>(&tfull[tb * C::kSplitN + half], tphase, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok)) goto epilogue_done;
        tc_fence_after();
        const uint32_t col_addr = lane_addr + static_cast<uint32_t>(tb * BN + g * CPW);
        // Two register buffers: the load of chunk c+1 is in flight while the
        // FMAs of chunk c run.
        uint32_t va[32], vb[32];
        tmem_ld_32x32b_x32(col_addr, va);
        tmem_ld_wait(va);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t(&cur)[32] = (c & 1) ? vb : va;
          uint32_t(&nxt)[32] = (c & 1) ? va : vb;
          if (c + 1 < NCH) tmem_ld_32x32b_x32(col_addr + 32 * (c + 1), nxt);
          if (c + 1 == NCH) {
            // Every load of this buffer has completed: hand it back to the MMA.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR) mbar_arrive_cluster(tb ? tempty_leader1 : tempty_leader0);
              else mbar_arrive(&tempty[tb * C::kSplitN + half]);
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            acc[c * 16 + j] = __ffma2_rn(
                make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])), scale2,
                acc[c * 16 + j]);
          if (c + 1 < NCH) tmem_ld_wait(nxt);
        }
        tb ^= 1;
        if (tb == 0) tphase ^= 1u;
      }
      const int64_t col0 = static_cast<int64_t>(t.n_tile) * BN + g * CPW;
      const int64_t slab0 = t.row0 + static_cast<int64_t>(rank) * BM + quad * 32;
      const bool slab_tma = slab0 < t.row_end && (!GROUPED || slab0 + 32 <= t.row_end);
      if (p.y_tma == 2 && slab_tma) {
        // FP32 split-K partials of split t.split, 16 columns per box.
        uint8_t* box = out_boxes + e * kOutBoxBytes;
#pragma unroll
        for (int c = 0; c < CPW / 16; ++c) {
          if (col0 + 16 * c >= p.N) break;
          uint32_t w16[16];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            w16[2 * j] = __float_as_uint(acc[c * 8 + j].x);
            w16[2 * j + 1] = __float_as_uint(acc[c * 8 + j].y);
          }
          store_out_box(&tmap_y, box, lane, w16, static_cast<int32_t>(col0 + 16 * c),
                        static_cast<int32_t>(slab0), t.split);
        }
      } else if (p.y_tma == 1 && slab_tma) {
        // Staged TMA stores; rows past M and columns past N are clipped.
        uint8_t* box = out_boxes + e * kOutBoxBytes;
#pragma unroll
        for (int c = 0; c < CPW / 32; ++c) {
          if (col0 + 32 * c >= p.N) break;
          uint32_t h[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) h[j] = pack_bf16x2(acc[c * 16 + j].x, acc[c * 16 + j].y);
          store_out_box(&tmap_y, box, lane, h, static_cast<int32_t>(col0 + 32 * c),
                        static_cast<int32_t>(slab0));
        }
      } else if (row_ok) {
        if (p.splits == 1) {
          __nv_bfloat16* yrow = p.y + row * p.N;
#pragma unroll
          for (int c = 0; c < CPW / 8; ++c) {
            const int64_t col = col0 + c * 8;
            if (vec_store && col + 8 <= p.N) {
              uint32_t h[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 b2 = __float22bfloat162_rn(acc[c * 4 + j]);
                h[j] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(yrow + col) = make_uint4(h[0], h[1], h[2], h[3]);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float v = (j & 1) ? acc[c * 4 + j / 2].y : acc[c * 4 + j / 2].x;
                if (col + j < p.N) yrow[col + j] = __float2bfloat16_rn(v);
              }
            }
          }
        } else {
          float* wrow = p.ws + (static_cast<int64_t>(t.split) * p.M + row) * p.N;
#pragma unroll
          for (int c = 0; c < CPW / 4; ++c) {
            const int64_t col = col0 + c * 4;
            const float2 lo = acc[2 * c], hi = acc[2 * c + 1];
            if ((p.N % 4) == 0 && col + 4 <= p.N) {
              *reinterpret_cast<float4*>(wrow + col) = make_float4(lo.x, lo.y, hi.x, hi.y);
            } else {
              const float v4[4] = {lo.x, lo.y, hi.x, hi.y};
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (col + j < p.N) wrow[col + j] = v4[j];
            }
          }
        }
      }
    }
  epilogue_done:
    if (lane == 0) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  // In pair mode neither CTA may release TMEM or exit while the other can
  // still touch its shared memory, barriers or TMEM.
  if (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace gemm
}  // namespace fp8bs
