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
// Roles (persistent CTAs, one per SM, walking work units in a fixed order;
// every control warp runs its loop with all 32 lanes and issues through
// elect.sync):
//   warp 0     TMA producer: A tile [ARows x 128] and W tile into a ring of
//              shared-memory stages (128B swizzle).
//   warp 1     MMA issuer and owner of the TMEM allocation.  With 192-wide
//              tiles and decode-sized A stages warp 3 issues too, the two
//              taking alternate K blocks.
//   warp 2     scale producer (and warp 3, on alternate K blocks, with
//              128-row A stages and 128- or 256-wide tiles): for its K
//              blocks it loads the 128 activation scales a_s[rows, kb] and
//              the weight scales w_s[nb, kb] of the tile (four of its steps
//              ahead, in registers) into a small shared-memory ring that the
//              epilogue reads.  The epilogue threads would otherwise each
//              wait on a scattered global load per K block, which measured
//              slower than the drain of the TMEM partial itself.
//   epilogue   8 warps from kFirstEpiWarp: warp w reads TMEM lanes
//              32*(w%4)..+31 (one output row per thread) and BN/2 columns
//              (column half (w - kFirstEpiWarp) / 4).  Loads of the next
//              32-column chunk overlap the FMAs of the current one.
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

#include "linear.cuh"
#include "quant.cuh"
#include "sm100.cuh"

namespace fp8bs {
namespace gemm {

constexpr int BM = 128;      // rows of A per CTA
constexpr int BK = 128;      // one K block per pipeline stage
constexpr int kMaxGroups = 1024;
// Ints of the grouped mode's table in shared memory (see group_table).
constexpr int kGroupTableInts = 2 * (kMaxGroups + 1);
#ifndef FP8BS_SPIN_WAITS
#define FP8BS_SPIN_WAITS 0
#endif
constexpr bool kSpinWaits = FP8BS_SPIN_WAITS != 0;

struct Params {
  const float* sa;          // [M_total, kbn]
  const float* sw;          // [G][nbn][kbn]
  __nv_bfloat16* y;         // [M_total, N]
  float* ws;                // [splits][M][N] FP32 partials when splits > 1; with
                            // out_f32 and one split, the FP32 output y itself
  const int64_t* m_offsets; // grouped mode: [G + 1] prefix row offsets (device)
  int64_t M;                // rows of A (M_total in grouped mode)
  int N;
  int kbn;                  // K / 128
  int nbn;                  // cdiv(N, 128)
  int m_tiles;              // dense mode: tiles of kUnitRows rows
  int n_group;              // dense mode, one split: tiles walk bands of n_group
                            // n tiles, m fastest inside a band (see tile_mn)
  int n_tiles;
  int splits;
  int kb_per_split;
  int num_units;            // dense mode; grouped mode derives it on the device
  int groups;               // grouped mode
  int y_tma;                // 1: bf16 y written by TMA stores through staging boxes;
                            // 2: FP32 split-K partials written by TMA stores (3-D map)
  // Split tail (dense mode, one split otherwise): units [0, full_units) are
  // whole tiles numbered as in the unsplit plan; the tail_tiles tiles after
  // them each become tail_splits units of tail_kbps K blocks whose FP32
  // partials go to tail_ws[(tail tile * tail_splits + split)][128][BN], summed
  // afterwards by tail_reduce_kernel.  tail_splits == 0: no split tail.
  int full_units;
  int tail_tiles;
  int tail_splits;
  int tail_kbps;
  float* tail_ws;
  // FP8 output (dense, BN = 256, one split): instead of storing y, the
  // epilogue rounds each row's 128-column block to bf16 and quantizes it as
  // act_quant would (q_out [M, N] e4m3 codes, s_out [M, N/128]); y (nullable)
  // then receives the bf16 values too.  With y_tma == 3, tmap_y maps q_out.
  uint8_t* q_out;
  float* s_out;
  int q_ue8m0;
  // FP32 output: y is stored unrounded, through the FP32 partial path (one
  // split: ws = y, y_tma 2 maps y as a single split; several: the reduction
  // writes FP32).  p.y is unused then.
  int out_f32;
  // Fused linear (FUSED instantiations): CTAs from gemm_ctas on quantize x
  // into fq_q / fq_s (the buffers tmap_a and sa read) and count the chunks
  // into fq_flags [m_tiles][kbn] (zero at launch); the GEMM CTAs wait for a
  // chunk's flag before reading its codes or scales.
  int gemm_ctas;
  int* fq_flags;
  uint8_t* fq_q;
  float* fq_s;
  int fq_ue8m0;
  // Test of the bounded waits only (0 in every product launch): CTA 0's scale
  // producer withholds its arrival for its K-block step stall_step - 1
  // (counted over its units from 0), so the epilogue's wait on that step
  // cannot complete and must give up.
  int stall_step;
};

// Nonzero unless v is a positive normal power of two.
__device__ __forceinline__ uint32_t not_pow2(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t e = (b >> 23) & 0xFFu;
  return (b & 0x807FFFFFu) | static_cast<uint32_t>(e == 0u) | static_cast<uint32_t>(e == 0xFFu);
}

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

// ARows: rows of A that one stage loads.  128 for M > 64; for decode-sized M
// (at most 16 or 64 rows) only those rows are loaded, so that the shared
// memory holds more stages of the weight stream, which bounds decode.  The MMA
// still reads a 128-row A operand: the rows past ARows come from the shared
// memory that follows the stage's A slot (the next A slots, then the W
// slots, all inside the CTA's allocation), and they only produce
// accumulator rows past M, which are never stored.
template <int BN, int ARows = 128>
struct Cfg {
  static_assert(BN == 128 || BN == 192 || BN == 256, "tile width");
  static_assert(ARows == 128 || ARows == 64 || ARows == 16, "A rows per stage");
  static constexpr int kABytes = ARows * BK;
  static constexpr int kBBytes = BN * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages =
      ARows == 128 ? (BN == 256 ? 4 : (BN == 192 ? 5 : 6))
                   : ((200 * 1024) / kStageBytes > 12 ? 12 : (200 * 1024) / kStageBytes);
  // Two epilogue warpgroups: each covers all 128 TMEM lanes (one warp per
  // 32-lane quadrant) and half of the tile's columns.
  static constexpr int kEpiWarps = 8;
  static constexpr int kColsPerWarp = BN / 2;
  static constexpr int kChunks = kColsPerWarp / 32;
  // Warps 0-3 form the control warpgroup (TMA, MMA, scales); for BN >= 192
  // it hands registers to the two epilogue warpgroups (setmaxnreg), for
  // BN = 128 every thread can hold its 64 accumulators at launch.
  // Weight blocks a tile's columns can touch: tiles start at multiples of BN,
  // so a 128- or 256-wide tile covers whole blocks and a 192-wide tile
  // straddles at most one block boundary.
  static constexpr int kNbSpan = BN == 128 ? 1 : 2;
  // The epilogue releases a TMEM buffer once its columns are in registers.
  // With at most 96 columns per thread (BN <= 192) all of them are loaded in
  // one batch, so the release comes one load latency after the MMA finishes;
  // with 128 (BN = 256) the registers only allow a two-deep chunk pipeline
  // whose FMAs delay the release.
  static constexpr bool kOneBatch = BN <= 192;
  static constexpr int kFirstEpiWarp = 4;
  static constexpr bool kSplitRegs = (BN >= 192);
  static constexpr int kCtrlRegs = 56;
  static constexpr int kEpiRegs = 224;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  // TMEM partial buffers: as many as the 512 columns hold (2 of 256 columns,
  // 4 of 128), so the epilogue can lag the tensor core by kAccBufs - 1 K blocks.
  static constexpr int kAccBufs = 512 / BN;
  // 128-row A stages with 256- or 128-wide tiles: warp 1 alone issues the
  // MMAs (about 400 cycles of issue per K block) and warps 2 and 3 both
  // produce scales, alternate K blocks each.  A producer's step is bound by
  // its load latency (~700-850 cycles); two of them keep the scales ahead
  // (measured on B200: 6-14 % faster at 128 x 256, 3-10 % at 128 x 128,
  // 9 % faster grouped GEMM).  192-wide tiles (384 cycles of MMA per K
  // block) and the decode stages (whose weight stream sets the pace; one
  // issuer measured 3 % slower there) keep two MMA warps (warps 1 and 3)
  // and one scale warp.
  static constexpr int kScaleWarps = (BN != 192 && ARows == 128) ? 2 : 1;
  static constexpr int kTmemCols = 512;
  static constexpr int kCtrlBytes = 512;
  // Scale ring: per K block the tile's 128 activation scales and its
  // (BN / 128) weight scales, or with row scales on W its BN column scales.
  static constexpr int kScaleSlots = 4;   // >= kAccBufs; slot b goes with TMEM buffer b
  static constexpr int kScaleSlotBytes = 4 * (BM + BN);
  static constexpr int kScaleBytes = kScaleSlots * kScaleSlotBytes;
  // grouped mode: per-group m-tile prefix (int)
  static constexpr int kGroupBytes = 4 * kGroupTableInts;
  // output staging boxes (one per epilogue warp), 1024-byte aligned
  __host__ __device__ static constexpr int out_offset(bool grouped) {
    return (kStages * kStageBytes + kCtrlBytes + kScaleBytes + (grouped ? kGroupBytes : 0) +
            1023) & ~1023;
  }
  __host__ __device__ static constexpr int smem_bytes(bool grouped) {
    return out_offset(grouped) + kEpiWarps * kOutBoxBytes + 1024;
  }
};

// Control block at the end of the tile ring.
template <int kStages>
struct Ctrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[4];     // TMEM partial buffer and its scale slot ready for the epilogue
  uint64_t tempty[4];    // TMEM partial buffer drained and its scale slot read
  uint64_t sempty[4];    // row scales on W: the epilogue is done with scale slot b
  uint64_t flush[2];     // per MMA issuer: all of its MMAs complete
  uint32_t tmem_base;
  int abort_flag;
  int num_units;
};

struct Unit {
  int64_t row0;      // first A/y row of the unit
  int64_t row_end;   // rows >= row_end are not stored
  int64_t w_row0;    // first W row (grouped: expert * N + n0)
  int group;
  int n_tile;
  int kb0, kb1;
  int split;
  int tail_slot;     // >= 0: FP32 partial slot of a split tail unit
};

// Dense units: m tile fastest, so the CTAs running at the same time share W
// tiles (and sweep all of A, which stays in L2).
// Tile t of a dense problem with one K split: bands of g = n_group n tiles
// (the last band narrower) are walked one after the other, and inside a band
// the m tile changes slowest, so the CTAs running at once share the band's
// W tiles (which stay in L2) while A streams once per band.  n_group = 1 is
// the m-fastest order (each W tile read once, A once per n tile), which suits
// an A small enough to stay in L2; a wide band suits a large A and a small W.
__host__ __device__ __forceinline__ void tile_mn(int tile, int m_tiles, int n_tiles, int g,
                                                 int& m_tile, int& n_tile) {
  const int band = tile / (m_tiles * g);
  const int width = min(g, n_tiles - band * g);
  const int rem = tile - band * m_tiles * g;
  m_tile = rem / width;
  n_tile = band * g + rem % width;
}

template <int kUnitRows>
__host__ __device__ __forceinline__ Unit dense_unit(const Params& p, int u) {
  Unit t;
  t.tail_slot = -1;
  if (p.tail_splits > 0 && u >= p.full_units) {
    // Split tail: consecutive units take different tiles, so the CTAs of the
    // last wave stream different operands.
    const int r = u - p.full_units;
    const int tt = r % p.tail_tiles;
    const int tile = p.full_units + tt;
    t.split = r / p.tail_tiles;
    int m_tile;
    tile_mn(tile, p.m_tiles, p.n_tiles, p.n_group, m_tile, t.n_tile);
    t.group = 0;
    t.row0 = static_cast<int64_t>(m_tile) * kUnitRows;
    t.row_end = p.M;
    t.kb0 = t.split * p.tail_kbps;
    t.kb1 = min(p.kbn, t.kb0 + p.tail_kbps);
    t.tail_slot = tt * p.tail_splits + t.split;
    return t;
  }
  int m_tile;
  if (p.splits == 1) {
    t.split = 0;
    tile_mn(u, p.m_tiles, p.n_tiles, p.n_group, m_tile, t.n_tile);
  } else {
    m_tile = u % p.m_tiles;
    const int rest = u / p.m_tiles;
    t.split = rest % p.splits;
    t.n_tile = rest / p.splits;
  }
  t.group = 0;
  t.row0 = static_cast<int64_t>(m_tile) * kUnitRows;
  t.row_end = p.M;
  t.kb0 = t.split * p.kb_per_split;
  t.kb1 = min(p.kbn, t.kb0 + p.kb_per_split);
  return t;
}

// Grouped units: n tile fastest inside one global m tile, so the CTAs running
// at the same time work on one or two experts and read each W_e once.
// The group table in shared memory: tile_prefix[g] (g <= G) is the number of
// m tiles of groups < g, and row_off[g] = tile_prefix[kMaxGroups + 1 + g]
// (g <= G) is the device offset g clamped to [0, M]; group g's rows are
// [row_off[g], max(row_off[g + 1], row_off[g])), the device offsets clamped to [0, M] and made non-decreasing.
// Built once per CTA by group_table, so that a unit's rows cost no global
// load on the producer's and the MMA issuers' paths.
__device__ __forceinline__ void group_table(const Params& p, int* table, int lane,
                                            int* num_units) {
  int* row_off = table + kMaxGroups + 1;
  for (int g = lane; g <= p.groups; g += 32) {
    int64_t o = __ldg(p.m_offsets + g);
    o = o < 0 ? 0 : (o > p.M ? p.M : o);
    row_off[g] = static_cast<int>(o);
  }
  __syncwarp();
  int carry = 0;
  for (int g0 = 0; g0 < p.groups; g0 += 32) {
    const int g = g0 + lane;
    int tiles = 0;
    if (g < p.groups) {
      const int lo = row_off[g], hi = max(row_off[g + 1], lo);
      tiles = (hi - lo + BM - 1) / BM;
    }
    int incl = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += v;
    }
    if (g < p.groups) table[g] = carry + incl - tiles;
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  if (lane == 0) {
    table[p.groups] = carry;
    *num_units = carry * p.n_tiles;
  }
}

template <int kUnitRows>
__host__ __device__ __forceinline__ Unit grouped_unit(const Params& p, const int* tile_prefix,
                                                      int u) {
  Unit t;
  const int gm = u / p.n_tiles;
  t.n_tile = u % p.n_tiles;
  int a = 0, b = p.groups;
  while (b - a > 1) {
    const int mid = (a + b) >> 1;
    if (tile_prefix[mid] <= gm) a = mid; else b = mid;
  }
  t.group = a;
  const int* row_off = tile_prefix + kMaxGroups + 1;
  const int64_t lo = row_off[a], hi = max(row_off[a + 1], row_off[a]);
  t.row0 = lo + static_cast<int64_t>(gm - tile_prefix[a]) * kUnitRows;
  t.row_end = hi;
  t.split = 0;
  t.tail_slot = -1;
  t.kb0 = 0;
  t.kb1 = p.kbn;
  return t;
}

// BROW: one scale per row of W (W column of y) and K block, as both operands
// of the weight-gradient GEMM carry (dense mode only).  Both scale tables are
// then read K-block-major, sa [K/128][M] and sw [K/128][N] (the host stages
// them so), which makes the scale producer's loads coalesced.  The
// scale producer then fills the slot with the tile's BN column scales, the
// epilogue multiplies a_s[row] by each column's scale before its FMA, and
// since those reads outlast the TMEM buffer's release, the slot has its own
// release barrier (sempty) that the producer waits on instead of tempty.
// CHECK: the caller promised power-of-two scales (a *_ue8m0 entry routed to
// this kernel, at decode-sized M): the first epilogue warp, before its first
// wait, reads the scales the CTA's units use and reports one that is not a
// positive normal power of two (device error 6).  Checked in the scale
// producer, the values slowed decode by ~5 us; in the TMA warp's spare lanes
// the divergent check ran ahead of the first TMA issue.  A compile-time
// switch, so the other instantiations carry none of it.
// FUSED: the fused linear layer (linear.cuh): CTAs from p.gemm_ctas on are
// quantizer CTAs reading x through tmap_x; the GEMM CTAs (dense, one K split,
// every unit within one wave) wait for each chunk's ready flag before they
// read its codes (TMA) and scales.  tmap_x is unused otherwise.
template <int BN, bool GROUPED, int ARows = 128, bool BROW = false, bool CHECK = false,
          bool FUSED = false>
__global__ void __launch_bounds__(Cfg<BN, ARows>::kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CUtensorMap tmap_y,
                    const __grid_constant__ CUtensorMap tmap_x, const Params p) {
  using C = Cfg<BN, ARows>;
  static_assert(!FUSED || (!GROUPED && !BROW && !CHECK && ARows == 128), "fused linear: dense GEMM");
  static_assert(!FUSED || C::smem_bytes(false) >= kQRingBytes + kQBarBytes + 1024,
                "quantizer ring fits the GEMM's shared memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  if (FUSED && static_cast<int>(blockIdx.x) >= p.gemm_ctas) {
    pdl_trigger();
    pdl_wait();
    const int qi = static_cast<int>(blockIdx.x) - p.gemm_ctas;
    const int nq = static_cast<int>(gridDim.x) - p.gemm_ctas;
    if (p.fq_ue8m0)
      quantize_cta<true>(&tmap_x, p.M, p.kbn * BK, p.fq_q, p.fq_s, p.fq_flags, smem, qi, nq);
    else
      quantize_cta<false>(&tmap_x, p.M, p.kbn * BK, p.fq_q, p.fq_s, p.fq_flags, smem, qi, nq);
    return;
  }
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + C::kStages * C::kABytes;
  Ctrl<C::kStages>* ctrl = reinterpret_cast<Ctrl<C::kStages>*>(smem + C::kStages * C::kStageBytes);
  static_assert(sizeof(Ctrl<C::kStages>) <= C::kCtrlBytes, "control block too large");
  uint64_t* full = ctrl->full;
  uint64_t* empty = ctrl->empty;
  uint64_t* tfull = ctrl->tfull;
  uint64_t* tempty = ctrl->tempty;
  uint64_t* sempty = ctrl->sempty;
  uint64_t* flush = ctrl->flush;
  static_assert(!(BROW && GROUPED), "row scales on W are a dense-mode variant");
  volatile int* abort_flag = &ctrl->abort_flag;
  float* scale_slots =
      reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + C::kCtrlBytes);
  int* tile_prefix = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes + C::kCtrlBytes +
                                            C::kScaleBytes);
  uint8_t* out_boxes = smem + C::out_offset(GROUPED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  const int unit_start = static_cast<int>(blockIdx.x);
  const int unit_step = FUSED ? p.gemm_ctas : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    // tfull[b] completes when the MMA's commit and the scale producer have
    // both arrived: the partial in TMEM buffer b and the scales of the same
    // K block in slot b are then ready, so the epilogue waits once per K block.
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&tfull[b], 2);
      mbar_init(&tempty[b], C::kEpiWarps);
      mbar_init(&sempty[b], C::kEpiWarps);
    }
    mbar_init(&flush[0], 1);
    mbar_init(&flush[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_descriptor(&tmap_a);
    tma_prefetch_descriptor(&tmap_w);
    if (p.y_tma) tma_prefetch_descriptor(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  // Inputs may come from the previous kernel of the stream (launched with
  // programmatic serialization): wait for it before any global access.
  pdl_wait();
  if (GROUPED) {
    // Clamp the device offsets to [0, M], count each group's m tiles and form
    // their exclusive prefix sum (warp 2, 32 groups per step).
    if (warp == 2) group_table(p, tile_prefix, lane, &ctrl->num_units);
  } else if (threadIdx.x == 0) {
    ctrl->num_units = p.num_units;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctrl->tmem_base;
  const int num_units = ctrl->num_units;

  auto unit_of = [&](int u) -> Unit {
    Unit t;
    if (GROUPED) {
      t = grouped_unit<BM>(p, tile_prefix, u);
      t.w_row0 = static_cast<int64_t>(t.group) * p.N + static_cast<int64_t>(t.n_tile) * BN;
    } else {
      t = dense_unit<BM>(p, u);
      t.w_row0 = static_cast<int64_t>(t.n_tile) * BN;
    }
    return t;
  };

  if (warp < C::kFirstEpiWarp) {
    if (C::kSplitRegs) reg_release<C::kCtrlRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the loop and takes the waits; one elected lane
    // issues the loads.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0;       // stages with a TMA load issued
    uint32_t armed_phase = 0; // parity each armed stage completes
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
        if (FUSED) {
          // The chunk's codes are written by a quantizer CTA of this launch.
          if (!__all_sync(0xFFFFFFFFu,
                          wait_chunk_flag(p.fq_flags + (t.row0 / BM) * p.kbn + kb, abort_flag)))
            goto producer_done;
          fence_proxy_async_global();
        }
        mbar_arrive_expect_tx_warp(&full[stage], C::kStageBytes);
        tma_load_2d_warp(a_tiles + stage * C::kABytes, &tmap_a, &full[stage], kb * BK,
                         static_cast<int32_t>(t.row0));
        tma_load_2d_warp(b_tiles + stage * C::kBBytes, &tmap_w, &full[stage], kb * BK,
                         static_cast<int32_t>(t.w_row0));
        armed |= 1u << stage;
        armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  producer_done:
    if (*abort_flag) {
      // Let every load in flight land before the CTA exits.
      for (int s = 0; s < C::kStages; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1 || (warp == 3 && C::kScaleWarps == 1)) {
    // ------------------------------------------------------------ MMA issuers
    // Two issuing warps: warp 1 takes the even and warp 3 the odd K blocks
    // of this CTA's sequence (i counts K blocks over all its units).  Each K
    // block writes a fresh partial into its own TMEM buffer and reads its own
    // stage, so the two streams need no ordering between them.  Each warp
    // walks its loop together and takes the waits; one elected lane issues.
    constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
    const uint32_t parity = warp == 1 ? 0u : 1u;
    uint32_t i = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      for (int kb = t.kb0; kb < t.kb1; ++kb, ++i) {
        if (C::kScaleWarps == 1 && (i & 1u) != parity) continue;
        const int stage = static_cast<int>(i % C::kStages);
        const uint32_t phase = (i / C::kStages) & 1u;
        const int tb = static_cast<int>(i % C::kAccBufs);
        const uint32_t tphase = (i / C::kAccBufs) & 1u;
        if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto mma_done;
        if (!mbar_wait_warp<kSpinWaits>(&tempty[tb], tphase ^ 1u, abort_flag)) goto mma_done;
        tc_fence_after();
        const uint32_t a_addr = smem_addr(a_tiles + stage * C::kABytes);
        const uint32_t b_addr = smem_addr(b_tiles + stage * C::kBBytes);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * BN);
#pragma unroll
        for (int k = 0; k < BK / 32; ++k)
          mma_f8f6f4_warp(d_tmem, smem_desc_k_sw128(a_addr + 32 * k),
                          smem_desc_k_sw128(b_addr + 32 * k), idesc, k > 0 ? 1u : 0u);
        mma_commit_warp(&tfull[tb]);
        mma_commit_warp(&empty[stage]);
      }
    }
  mma_done:
    // Every MMA this warp issued must finish before the TMEM columns are
    // released.
    mma_commit_warp(&flush[parity]);
    mbar_wait(&flush[parity], 0, nullptr);
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ scale producer(s)
    // Walks the same (unit, K block) sequence as the epilogue (with two
    // scale warps, each its alternate steps).  A second cursor runs kAhead
    // of its steps ahead and loads the scales into a ring of registers.
    // (The warp barrier and the release before each arrival wait for the
    // lane's loads in flight, so a warp's step costs about one load latency,
    // ~700-850 cycles measured on B200; hence two warps where a K block's
    // MMAs take less.)  Step i uses the slot of its TMEM buffer,
    // i % kAccBufs, once the epilogue has released that buffer (tempty), and
    // then arrives on its tfull: a_s of the tile's 128 rows (0 past the last
    // row) and w_s of the weight blocks the tile touches (0 past the last),
    // or with BROW the scales of the tile's BN columns (0 past the last), in
    // which case the slot is reused once the epilogue has read it (sempty).
    // With BROW the ring holds BN / 32 more values per step; two steps ahead
    // (over a microsecond of MMA work) keep it within the producer's registers.
    constexpr int kAhead = BROW ? 2 : 4;
    constexpr int kNbPerTile = C::kNbSpan;
    constexpr int kWRegs = BROW ? BN / 32 : 1;
    uint64_t* slot_free = BROW ? sempty : tempty;
    struct Cursor {
      int u, kb, kb1, group, nb0, n0;
      int64_t row0, row_end;
      bool valid;
    };
    auto begin = [&](Cursor& c, int u) {
      c.u = u;
      c.valid = u < num_units;
      if (c.valid) {
        const Unit t = unit_of(u);
        c.kb = t.kb0;
        c.kb1 = t.kb1;
        c.group = t.group;
        c.nb0 = (t.n_tile * BN) / 128;
        c.n0 = t.n_tile * BN;
        c.row0 = t.row0;
        c.row_end = t.row_end;
      }
    };
    auto next = [&](Cursor& c) {
      if (c.valid && ++c.kb >= c.kb1) begin(c, c.u + unit_step);
    };
    auto load = [&](const Cursor& c, float (&va)[4], float (&vw)[kWRegs]) {
      if (FUSED && c.valid) {
        // The scales are written in this launch: wait for the chunk, then read
        // them from L2 (not through the non-coherent read-only path).
        wait_chunk_flag(p.fq_flags + (c.row0 / BM) * p.kbn + c.kb, abort_flag);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t row = c.row0 + lane + 32 * j;
          va[j] = row < c.row_end ? __ldcg(p.sa + row * p.kbn + c.kb) : 0.0f;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t row = c.row0 + lane + 32 * j;
          va[j] = (c.valid && row < c.row_end)
                      ? __ldg(BROW ? p.sa + c.kb * p.M + row : p.sa + row * p.kbn + c.kb)
                      : 0.0f;
        }
      }
      if (BROW) {
        // K-block-major tables (sa [kbn][M], sw [kbn][N]): lanes read
        // consecutive rows / columns, one coalesced load per 32 values.
#pragma unroll
        for (int j = 0; j < kWRegs; ++j) {
          const int64_t col = c.n0 + lane + 32 * j;
          vw[j] = (c.valid && col < p.N) ? __ldg(p.sw + c.kb * static_cast<int64_t>(p.N) + col) : 0.0f;
        }
      } else {
        const int nb = c.nb0 + lane;
        vw[0] = (c.valid && lane < kNbPerTile && nb < p.nbn)
                    ? __ldg(p.sw + (static_cast<int64_t>(c.group) * p.nbn + nb) * p.kbn + c.kb)
                    : 0.0f;
      }
    };
    // With two scale warps, warp 2 takes the even and warp 3 the odd steps
    // of the sequence; each cursor then moves NP K blocks per step.
    constexpr int NP = C::kScaleWarps;
    const int pi = (NP == 2 && warp == 3) ? 1 : 0;
    float ra[kAhead][4], rw[kAhead][kWRegs];
    Cursor ahead, cur;
    begin(ahead, unit_start);
    begin(cur, unit_start);
    if (pi) {
      next(ahead);
      next(cur);
    }
#pragma unroll
    for (int d = 0; d < kAhead; ++d) {
      load(ahead, ra[d], rw[d]);
#pragma unroll
      for (int k = 0; k < NP; ++k) next(ahead);
    }
    const uint32_t stall_at =
        (p.stall_step > 0 && blockIdx.x == 0) ? static_cast<uint32_t>(p.stall_step - 1) : 0xFFFFFFFFu;
    uint32_t step = static_cast<uint32_t>(pi);
    // Step `step` uses the slot of its TMEM buffer, step % kAccBufs, with
    // phase (step / kAccBufs) & 1.  (Kept as a running pair with one scale
    // warp, recomputed with two: each form is the one that compiles without
    // spills in the 56 registers of the control warps.)
    static_assert(NP <= C::kAccBufs, "scale warps per TMEM buffer");
    int slot_run = pi;
    uint32_t sphase_run = 0;
    while (cur.valid) {
#pragma unroll
      for (int ph = 0; ph < kAhead; ++ph) {
        if (!cur.valid) break;
        const int slot = NP == 1 ? slot_run : static_cast<int>(step % C::kAccBufs);
        const uint32_t sphase = NP == 1 ? sphase_run : (step / C::kAccBufs) & 1u;
        const bool ok = mbar_wait(&slot_free[slot], sphase ^ 1u, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok)) goto scales_done;
        float* dst = scale_slots + slot * (C::kScaleSlotBytes / 4);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[lane + 32 * j] = ra[ph][j];
        if (BROW) {
#pragma unroll
          for (int j = 0; j < kWRegs; ++j) dst[BM + lane + 32 * j] = rw[ph][j];
        } else if (lane < kNbPerTile) {
          dst[BM + lane] = rw[ph][0];
        }
        __syncwarp();
        if (lane == 0 && step != stall_at) mbar_arrive(&tfull[slot]);
        step += NP;
        if (NP == 1 && ++slot_run == C::kAccBufs) {
          slot_run = 0;
          sphase_run ^= 1u;
        }
        load(ahead, ra[ph], rw[ph]);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          next(ahead);
          next(cur);
        }
      }
    }
  scales_done:
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
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    if (CHECK && !GROUPED && e == 0) {
      // Before its first wait, which at decode-sized M comes microseconds
      // before the first partial: a_s [M, kbn] (small there) is shared out
      // over the CTAs, and each CTA checks the w_s blocks of its own units,
      // four independent loads per lane in flight at a time.
      uint32_t bad = 0;
      const int64_t na = p.M * p.kbn;
      const int64_t step_a = static_cast<int64_t>(gridDim.x) * 32;
      for (int64_t i = static_cast<int64_t>(blockIdx.x) * 32 + lane; i < na; i += 4 * step_a) {
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = i + j * step_a < na ? __ldg(p.sa + i + j * step_a) : 1.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) bad |= not_pow2(v[j]);
      }
      for (int u = unit_start; u < num_units; u += unit_step) {
        const Unit t = unit_of(u);
        const int nb0 = (t.n_tile * BN) / 128;
        const int nkb = t.kb1 - t.kb0;
        const int cnt = C::kNbSpan * nkb;
        for (int i = lane; i < cnt; i += 4 * 32) {
          float v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int el = i + 32 * j;
            const int nb = nb0 + el / nkb;
            v[j] = (el < cnt && nb < p.nbn)
                       ? __ldg(p.sw + static_cast<int64_t>(nb) * p.kbn + t.kb0 + el % nkb)
                       : 1.0f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) bad |= not_pow2(v[j]);
        }
      }
      if (__any_sync(0xFFFFFFFFu, bad != 0u) && lane == 0) report_error(6);
    }
    const bool vec_store = (p.N % 8) == 0;
    int tb = 0;
    uint32_t tphase = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      const int64_t row = t.row0 + row_in_tile;
      const bool row_ok = row < t.row_end;
      // Weight block of each 32-column chunk of this warp, relative to the
      // tile's first block (chunks never straddle a block boundary).
      const int nb0 = (t.n_tile * BN) / 128;
      int nb_of[NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) nb_of[c] = ((t.n_tile * BN + g * CPW + 32 * c) >> 7) - nb0;
      float2 acc[CPW / 2];
#pragma unroll
      for (int j = 0; j < CPW / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
      // A warp whose 32 rows all lie past the unit's end (decode-sized M, an
      // expert's last m tile) loads and accumulates nothing; it only takes
      // the waits and releases.  Dense prefill tiles compile without the
      // test: measured on B200, its branch cost the 256-wide dense kernel
      // 2-5 %, while it made decode 4-7 % and the grouped GEMM 6 % faster.
      const bool live = (ARows == 128 && !GROUPED) || t.row0 + quad * 32 < t.row_end;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const bool ok = mbar_wait<kSpinWaits>(&tfull[tb], tphase, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok)) goto epilogue_done;
        tc_fence_after();
        if (!live) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&tempty[tb]);
            if (BROW) mbar_arrive(&sempty[tb]);
          }
          if (++tb == C::kAccBufs) {
            tb = 0;
            tphase ^= 1u;
          }
          continue;
        }
        // This K block's scale products a_s[row, kb] * w_s[nb, kb], read before
        // the buffer (and with it the scale slot) is released below.
        const float* src = scale_slots + tb * (C::kScaleSlotBytes / 4);
        const float sa_row = src[row_in_tile];
        float scale_nb[C::kNbSpan];
#pragma unroll
        for (int i = 0; i < C::kNbSpan; ++i) scale_nb[i] = sa_row * src[BM + i];
        // BROW: this warp's column scales (the slot stays valid until sempty).
        const float* sb_col = src + BM + g * CPW;
        const float2 sa2 = make_float2(sa_row, sa_row);
        const uint32_t col_addr = lane_addr + static_cast<uint32_t>(tb * BN + g * CPW);
        if (C::kOneBatch) {
          // All of this warp's columns in one batch, then hand the buffer back
          // to the MMA before the FMAs.
          uint32_t v[NCH][32];
#pragma unroll
          for (int c = 0; c < NCH; ++c) tmem_ld_32x32b_x32(col_addr + 32 * c, v[c]);
#pragma unroll
          for (int c = 0; c < NCH; ++c) tmem_ld_wait(v[c]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[tb]);
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const float sc = C::kNbSpan == 1 ? scale_nb[0] : (nb_of[c] ? scale_nb[C::kNbSpan - 1] : scale_nb[0]);
            const float2 scale2 = make_float2(sc, sc);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              // BROW: four column scales per 16-byte (broadcast) read
              float2 s_lo = scale2, s_hi = scale2;
              if (BROW) {
                const float4 sb4 = *reinterpret_cast<const float4*>(sb_col + 32 * c + 2 * j);
                s_lo = __fmul2_rn(sa2, make_float2(sb4.x, sb4.y));
                s_hi = __fmul2_rn(sa2, make_float2(sb4.z, sb4.w));
              }
              acc[c * 16 + j] = __ffma2_rn(
                  make_float2(__uint_as_float(v[c][2 * j]), __uint_as_float(v[c][2 * j + 1])),
                  s_lo, acc[c * 16 + j]);
              acc[c * 16 + j + 1] = __ffma2_rn(
                  make_float2(__uint_as_float(v[c][2 * j + 2]), __uint_as_float(v[c][2 * j + 3])),
                  s_hi, acc[c * 16 + j + 1]);
            }
          }
        } else {
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
              if (lane == 0) mbar_arrive(&tempty[tb]);
            }
            const float sc = C::kNbSpan == 1 ? scale_nb[0] : (nb_of[c] ? scale_nb[C::kNbSpan - 1] : scale_nb[0]);
            const float2 scale2 = make_float2(sc, sc);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              float2 s_lo = scale2, s_hi = scale2;
              if (BROW) {
                const float4 sb4 = *reinterpret_cast<const float4*>(sb_col + 32 * c + 2 * j);
                s_lo = __fmul2_rn(sa2, make_float2(sb4.x, sb4.y));
                s_hi = __fmul2_rn(sa2, make_float2(sb4.z, sb4.w));
              }
              acc[c * 16 + j] = __ffma2_rn(
                  make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])),
                  s_lo, acc[c * 16 + j]);
              acc[c * 16 + j + 1] = __ffma2_rn(
                  make_float2(__uint_as_float(cur[2 * j + 2]), __uint_as_float(cur[2 * j + 3])),
                  s_hi, acc[c * 16 + j + 1]);
            }
            if (c + 1 < NCH) tmem_ld_wait(nxt);
          }
        }
        if (BROW) {
          // Done with this K block's column scales: the producer may refill the slot.
          __syncwarp();
          if (lane == 0) mbar_arrive(&sempty[tb]);
        }
        if (++tb == C::kAccBufs) {
          tb = 0;
          tphase ^= 1u;
        }
      }
      if (!GROUPED && BN == 256 && p.q_out != nullptr) {
        // FP8 output: this thread's 128 columns of its row are one 1x128
        // block of y.  Same steps as act_quant on the bf16 y: round to bf16,
        // amax over the bf16 values, s = block_scale(amax), q = e4m3(y / s).
        const int64_t col0 = static_cast<int64_t>(t.n_tile) * BN + g * CPW;
        if (col0 < p.N) {
          uint32_t hb[CPW / 2];
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < CPW / 2; ++j) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[j].x, acc[j].y);
            hb[j] = *reinterpret_cast<const uint32_t*>(&b2);
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(hb[j] << 16)),
                                     fabsf(__uint_as_float(hb[j] & 0xFFFF0000u))));
          }
          const float sc = block_scale(amax, p.q_ue8m0 != 0);
          const float r = __frcp_rn(sc);
          uint32_t codes[CPW / 4];
#pragma unroll
          for (int h = 0; h < CPW / 8; ++h) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              v[2 * j] = __uint_as_float(hb[4 * h + j] << 16);
              v[2 * j + 1] = __uint_as_float(hb[4 * h + j] & 0xFFFF0000u);
            }
            const uint2 c = p.q_ue8m0 ? quantize8<true>(v, sc, r) : quantize8<false>(v, sc, r);
            codes[2 * h] = c.x;
            codes[2 * h + 1] = c.y;
          }
          if (row_ok) p.s_out[row * (p.N / 128) + col0 / 128] = sc;
          const int64_t slab0 = t.row0 + quad * 32;
          if (p.y_tma == 3 && slab0 < t.row_end) {
            uint8_t* box = out_boxes + e * kOutBoxBytes;
#pragma unroll
            for (int c = 0; c < CPW / 64; ++c)
              store_out_box(&tmap_y, box, lane, *reinterpret_cast<const uint32_t(*)[16]>(&codes[16 * c]),
                            static_cast<int32_t>(col0 + 64 * c), static_cast<int32_t>(slab0));
          } else if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(p.q_out + row * p.N + col0);
#pragma unroll
            for (int c = 0; c < CPW / 16; ++c)
              dst[c] = make_uint4(codes[4 * c], codes[4 * c + 1], codes[4 * c + 2], codes[4 * c + 3]);
          }
          if (p.y != nullptr && row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(p.y + row * p.N + col0);
#pragma unroll
            for (int c = 0; c < CPW / 8; ++c)
              dst[c] = make_uint4(hb[4 * c], hb[4 * c + 1], hb[4 * c + 2], hb[4 * c + 3]);
          }
        }
        continue;
      }
      if (!GROUPED && t.tail_slot >= 0) {
        // FP32 partial of a split tail unit: the whole 128 x BN tile, rows and
        // columns past the matrix included (the reduction masks them).
        float* dst = p.tail_ws + (static_cast<int64_t>(t.tail_slot) * BM + row_in_tile) * BN + g * CPW;
#pragma unroll
        for (int c = 0; c < CPW / 4; ++c)
          *reinterpret_cast<float4*>(dst + 4 * c) =
              make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
        continue;
      }
      const int64_t col0 = static_cast<int64_t>(t.n_tile) * BN + g * CPW;
      const int64_t slab0 = t.row0 + quad * 32;
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
        if (p.splits == 1 && !p.out_f32) {
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Sum of the FP32 partials of the split tail tiles, in split order, into y
// (bf16, rounded to nearest even, or FP32).  One thread per 4 consecutive
// columns of one tile row.
template <typename OutT>
__global__ void __launch_bounds__(256)
    tail_reduce_kernel(const float* __restrict__ ws, OutT* __restrict__ y, int64_t M,
                       int N, int m_tiles, int n_tiles, int n_group, int full_units,
                       int tail_tiles, int splits, int bn) {
  pdl_trigger();
  pdl_wait();
  const int groups = bn / 4;
  const int64_t items = static_cast<int64_t>(tail_tiles) * BM * groups;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < items;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    const int tt = static_cast<int>(i / (BM * groups));
    const int rem = static_cast<int>(i - static_cast<int64_t>(tt) * BM * groups);
    const int r = rem / groups, c = (rem - r * groups) * 4;
    int m_tile, n_tile;
    tile_mn(full_units + tt, m_tiles, n_tiles, n_group, m_tile, n_tile);
    const int64_t row = static_cast<int64_t>(m_tile) * BM + r;
    const int64_t col = static_cast<int64_t>(n_tile) * bn + c;
    if (row >= M || col >= N) continue;
    float4 s = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int sp = 0; sp < splits; ++sp) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(
          ws + ((static_cast<int64_t>(tt) * splits + sp) * BM + r) * bn + c));
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    OutT* dst = y + row * N + col;
    const float v4[4] = {s.x, s.y, s.z, s.w};
    if constexpr (std::is_same_v<OutT, float>) {
      if ((N % 4) == 0 && col + 4 <= N) {
        *reinterpret_cast<float4*>(dst) = s;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col + j < N) dst[j] = v4[j];
      }
    } else if ((N % 4) == 0 && col + 4 <= N) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&lo);
      u.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(dst) = u;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (col + j < N) dst[j] = __float2bfloat16_rn(v4[j]);
    }
  }
}

}  // namespace gemm
}  // namespace fp8bs
