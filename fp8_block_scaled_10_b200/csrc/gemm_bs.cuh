// Block-scaled FP8 GEMM for ue8m0 scales (Blackwell tcgen05.mma
// kind::mxf8f6f4.block_scale): the same y = A * W^T as fp8_gemm_kernel, for
// the case where every activation scale a_s[m, kb] and weight scale
// w_s[nb, kb] is a positive power of two ("Understanding Dynamic and Static
// Activation Quantization Schemes in DeepSeek-V3", section "How Dynamic
// Activation Quantization Works": scale_fmt "ue8m0" rounds scales to powers of
// two for hardware compatibility).
//
// A power-of-two scale is exactly an 8-bit exponent, which the tensor core
// applies itself: each MMA of K = 32 multiplies row m of A by 2^(e_a[m]-127)
// and row n of W by 2^(e_w[n]-127) before accumulating in FP32.  The
// accumulator therefore runs over the whole K range of a tile in TMEM, with
// no per-K-block promotion: the epilogue reads TMEM once per tile.
//
// Scale factors in TMEM: for every 128 rows and a group of four consecutive
// 128-wide K blocks 4g .. 4g + 3, a 512-byte atom whose byte
// 16*(r%32) + 4*(r/32) + j holds the exponent of row r for K block 4g + j,
// copied from shared memory by tcgen05.cp 32x128b.warpx4 into 4 TMEM
// columns.  Each of the four MMAs (K = 32) of K block 4g + j selects byte j
// of its scale cells (the scale factor id of the instruction descriptor):
// one scale covers all 128 K elements of the block.  One copy per four K
// blocks: measured on B200, three copies per K block (one per atom) kept the
// tensor pipe busy 778 cycles per K block against 512 for the MMAs alone.
//
// Roles (persistent, one CTA per SM, 12 warps; the TMA and MMA warps run
// their loops with all 32 lanes and issue through elect.sync):
//   warp 0      TMA producer of A [128 x 128] and W [BN x 128] tiles.
//   warp 1      TMEM owner; copies each K-block group's scale atoms into a
//               TMEM ring and issues the block-scaled MMAs.
//   warp 2      scale producer: reads a_s / w_s for one K-block group at a
//               time, writes the exponent atoms into a shared-memory ring
//               of kSFSlots groups and checks that each scale is a positive
//               normal power of two (else device error FP8BS_ERR_SCALE = 6).
//   warps 4-11  epilogue: per tile, each thread reads one row of BN/2
//               accumulator columns into registers as bf16, releases the
//               accumulator, then stores (or writes FP32 split-K partials).
#pragma once

#include "gemm.cuh"

namespace fp8bs {
namespace gemm {

template <int BN>
struct BsCfg {
  static constexpr int kABytes = BM * BK;
  static constexpr int kBBytes = BN * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;   // TMA bytes per stage
  static constexpr int kSFAtoms = 1 + BN / 128;           // one for A, BN/128 for W
  static constexpr int kSFBytes = 512 * kSFAtoms;         // one K-block group's atoms
  static constexpr int kSFGroup = 4;                      // K blocks per scale atom
  static constexpr int kSFSlots = 3;                      // groups in flight (smem and TMEM)
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kAccBufs = (BN == 256) ? 1 : 2;    // TMEM accumulators
  static constexpr int kSFCols = 4 * kSFAtoms;            // TMEM columns per group slot
  static constexpr int kSFBase = kAccBufs * BN;
  static constexpr int kTmemCols = 512;
  static_assert(kSFBase + kSFSlots * kSFCols <= kTmemCols, "TMEM budget");
  static constexpr int kEpiWarps = 8;
  static constexpr int kColsPerWarp = BN / 2;
  static constexpr int kFirstEpiWarp = 4;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr int kCtrlBytes = 256;
  static constexpr int kGroupBytes = 4 * kGroupTableInts;
  __host__ __device__ static constexpr int out_offset(bool grouped) {
    return (kStages * kStageBytes + kSFSlots * kSFBytes + kCtrlBytes +
            (grouped ? kGroupBytes : 0) + 1023) &
           ~1023;
  }
  __host__ __device__ static constexpr int smem_bytes(bool grouped) {
    return out_offset(grouped) + kEpiWarps * kOutBoxBytes + 1024;
  }
};

template <int kStages>
struct BsCtrl {
  uint64_t full[kStages];    // TMA bytes
  uint64_t empty[kStages];
  uint64_t sffull[3];        // scale-group slot written (the scale producer)
  uint64_t sfempty[3];       // scale-group slot's MMAs complete (commit)
  uint64_t tfull[2];         // accumulator ready for the epilogue
  uint64_t tempty[2];        // accumulator drained
  uint64_t flush;
  uint32_t tmem_base;
  int abort_flag;
  int num_units;
};

// Exponent byte of a ue8m0 scale; *bad is set unless v is a positive normal
// power of two.
__device__ __forceinline__ uint32_t ue8m0_byte(float v, bool* bad) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t e = (b >> 23) & 0xFFu;
  if ((b & 0x807FFFFFu) != 0u || e == 0u || e == 0xFFu) *bad = true;
  return e;
}

// BROW: one scale per row of W and K block (dense mode), the second operand
// of the weight-gradient GEMM; the W atoms then hold a scale per row, laid
// out like A's, instead of one block scale repeated.  Both scale tables are
// then read K-block-major, sa [K/128][M] and sw [K/128][N], as the host
// stages them.
template <int BN, bool GROUPED, bool BROW = false>
__global__ void __launch_bounds__(BsCfg<BN>::kThreads, 1)
    fp8_gemm_bs_kernel(const __grid_constant__ CUtensorMap tmap_a,
                       const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  using C = BsCfg<BN>;
  static_assert(!(BROW && GROUPED), "row scales on W are a dense-mode variant");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_tiles = smem;
  uint8_t* b_tiles = smem + C::kStages * C::kABytes;
  uint8_t* sf_tiles = smem + C::kStages * C::kStageBytes;
  BsCtrl<C::kStages>* ctrl =
      reinterpret_cast<BsCtrl<C::kStages>*>(sf_tiles + C::kSFSlots * C::kSFBytes);
  static_assert(C::kSFSlots <= 3, "scale-group barriers");
  static_assert(sizeof(BsCtrl<C::kStages>) <= C::kCtrlBytes, "control block too large");
  uint64_t* full = ctrl->full;
  uint64_t* empty = ctrl->empty;
  uint64_t* tfull = ctrl->tfull;
  uint64_t* tempty = ctrl->tempty;
  uint64_t* flush = &ctrl->flush;
  uint64_t* sffull = ctrl->sffull;
  uint64_t* sfempty = ctrl->sfempty;
  volatile int* abort_flag = &ctrl->abort_flag;
  int* tile_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(ctrl) + C::kCtrlBytes);
  uint8_t* out_boxes = smem + C::out_offset(GROUPED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  const int unit_start = static_cast<int>(blockIdx.x);
  const int unit_step = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int g = 0; g < C::kSFSlots; ++g) {
      mbar_init(&sffull[g], 1);
      mbar_init(&sfempty[g], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kEpiWarps);
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
    tmem_alloc(&ctrl->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  // Inputs may come from the previous kernel of the stream (launched with
  // programmatic serialization): wait for it before any global access.
  pdl_wait();
  if (GROUPED) {
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the loop; one elected lane issues.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_phase = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
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
      for (int s = 0; s < C::kStages; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale producer
    // Walks this CTA's (unit, K-block group) sequence.  Group q covers the K
    // blocks 4q .. 4q + 3 (those outside the unit or past K are never used by
    // an MMA; they get exponent 127, a scale of 1).  For every group it loads
    // the scales first, all at once from clamped (always valid) indices so
    // that their latencies overlap, then waits until the MMAs that read the
    // slot's previous group have completed and writes the atoms: row r of A
    // (lane + 32 j) and of W (its block's scale, or with BROW its own row
    // scale), one exponent byte per K block.  A fence makes them visible to
    // the tensor core's copy before the arrival on sffull.
    constexpr int kG = C::kSFGroup;
    constexpr int kWA = BN / 128;   // W atoms
    bool bad = false;
    uint32_t gi = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      const int nb0 = (t.n_tile * BN) / 128;
      const int64_t n0 = t.w_row0 - static_cast<int64_t>(t.group) * p.N;   // first W row (column of y)
      for (int q = t.kb0 / kG; q <= (t.kb1 - 1) / kG; ++q, ++gi) {
        const int slot = static_cast<int>(gi % C::kSFSlots);
        int kbc[kG];
        bool kin[kG];
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          const int kb = q * kG + j;
          kin[j] = kb >= t.kb0 && kb < t.kb1;
          kbc[j] = kb < t.kb0 ? t.kb0 : (kb >= t.kb1 ? t.kb1 - 1 : kb);
        }
        float va[4][kG];
        bool rin[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int64_t row = t.row0 + lane + 32 * r;
          rin[r] = row < t.row_end;
          const int64_t rc = rin[r] ? row : t.row_end - 1;
#pragma unroll
          for (int j = 0; j < kG; ++j)
            va[r][j] = __ldg(BROW ? p.sa + static_cast<int64_t>(kbc[j]) * p.M + rc
                                  : p.sa + rc * p.kbn + kbc[j]);
        }
        constexpr int kWR = BROW ? 4 : 1;   // W rows per lane and atom
        float vw[kWA][kWR][kG];
        bool win[kWA][kWR];
#pragma unroll
        for (int a = 0; a < kWA; ++a) {
#pragma unroll
          for (int r = 0; r < kWR; ++r) {
            const float* src;
            if (BROW) {
              const int64_t n = n0 + 128 * a + lane + 32 * r;
              win[a][r] = n < p.N;
              src = p.sw + (win[a][r] ? n : p.N - 1);
            } else {
              const int nb = nb0 + a;
              win[a][r] = nb < p.nbn;
              src = p.sw + (static_cast<int64_t>(t.group) * p.nbn + (win[a][r] ? nb : p.nbn - 1)) * p.kbn;
            }
#pragma unroll
            for (int j = 0; j < kG; ++j)
              vw[a][r][j] = __ldg(src + static_cast<int64_t>(kbc[j]) * (BROW ? p.N : 1));
          }
        }
        const bool ok = mbar_wait(&sfempty[slot], ((gi / C::kSFSlots) & 1u) ^ 1u, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok)) goto scales_done;
        // Exponent word of one row: byte j = K block q * kG + j.
        auto word = [&](const float (&v)[kG], bool row_in) -> uint32_t {
          uint32_t w = 0;
#pragma unroll
          for (int j = 0; j < kG; ++j) {
            const uint32_t e = ue8m0_byte(v[j], &bad);
            w |= (row_in && kin[j] ? e : 127u) << (8 * j);
          }
          return w;
        };
        uint8_t* atoms = sf_tiles + slot * C::kSFBytes;
        *reinterpret_cast<uint4*>(atoms + 16 * lane) =
            make_uint4(word(va[0], rin[0]), word(va[1], rin[1]), word(va[2], rin[2]),
                       word(va[3], rin[3]));
#pragma unroll
        for (int a = 0; a < kWA; ++a) {
          uint4 w4;
          if (BROW) {
            w4 = make_uint4(word(vw[a][0], win[a][0]), word(vw[a][kWR > 1 ? 1 : 0], win[a][kWR > 1 ? 1 : 0]),
                            word(vw[a][kWR > 2 ? 2 : 0], win[a][kWR > 2 ? 2 : 0]),
                            word(vw[a][kWR > 3 ? 3 : 0], win[a][kWR > 3 ? 3 : 0]));
          } else {
            const uint32_t w = word(vw[a][0], win[a][0]);
            w4 = make_uint4(w, w, w, w);
          }
          *reinterpret_cast<uint4*>(atoms + 512 * (1 + a) + 16 * lane) = w4;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sffull[slot]);
      }
    }
  scales_done:
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report_error(6);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop and takes the waits; one elected lane
    // issues the copies, MMAs and commits.
    constexpr uint32_t idesc = idesc_e4m3_block_scaled(BM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int tb = 0;
    uint32_t tphase = 0;
    uint32_t gi = 0;   // K-block groups started
    uint32_t tsf = 0;  // TMEM scale slot of the current group
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      // The epilogue has drained this accumulator (tile u - 2 * step).
      if (!mbar_wait_warp(&tempty[tb], tphase ^ 1u, abort_flag)) goto mma_done;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * BN);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const int slot = static_cast<int>(gi % C::kSFSlots);
        if (kb == t.kb0 || kb % C::kSFGroup == 0) {
          // A new K-block group: its scale atoms into the slot's TMEM
          // columns (A, then W), once for the group's K blocks.
          if (!mbar_wait_warp(&sffull[slot], (gi / C::kSFSlots) & 1u, abort_flag)) goto mma_done;
          tc_fence_after();
          tsf = tmem_base + static_cast<uint32_t>(C::kSFBase + slot * C::kSFCols);
          const uint8_t* atoms = sf_tiles + slot * C::kSFBytes;
#pragma unroll
          for (int a = 0; a < C::kSFAtoms; ++a)
            tmem_copy_32x128b_x4_warp(tsf + 4 * a, smem_desc_rows16(smem_addr(atoms + 512 * a)));
        }
        if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto mma_done;
        tc_fence_after();
        const uint32_t a_addr = smem_addr(a_tiles + stage * C::kABytes);
        const uint32_t b_addr = smem_addr(b_tiles + stage * C::kBBytes);
        // Byte kb % 4 of every scale cell is this K block's exponent, for
        // all four K = 32 slices of the block.
        const uint32_t sub = static_cast<uint32_t>(kb % C::kSFGroup);
#pragma unroll
        for (int k = 0; k < BK / 32; ++k)
          mma_mxf8_block_scaled_warp(d_tmem, smem_desc_k_sw128(a_addr + 32 * k),
                                     smem_desc_k_sw128(b_addr + 32 * k),
                                     idesc | (sub << 29) | (sub << 4), tsf | (sub << 30),
                                     (tsf + 4) | (sub << 30), (kb > t.kb0 || k > 0) ? 1u : 0u);
        mma_commit_warp(&empty[stage]);
        if (kb + 1 == t.kb1 || kb % C::kSFGroup == C::kSFGroup - 1) {
          // The group's last MMAs: its slot is free once they complete.
          mma_commit_warp(&sfempty[slot]);
          ++gi;
        }
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      mma_commit_warp(&tfull[tb]);
      if (++tb == C::kAccBufs) {
        tb = 0;
        tphase ^= 1u;
      }
    }
  mma_done:
    mma_commit_warp(flush);
    mbar_wait(flush, 0, nullptr);
    __syncwarp();
  } else if (warp >= C::kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::kFirstEpiWarp;
    const int quad = warp & 3;
    const int g = e >> 2;
    constexpr int CPW = C::kColsPerWarp;
    constexpr int NCH = CPW / 32;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const bool vec_store = (p.N % 8) == 0;
    int tb = 0;
    uint32_t tphase = 0;
    for (int u = unit_start; u < num_units; u += unit_step) {
      const Unit t = unit_of(u);
      const bool ok = mbar_wait(&tfull[tb], tphase, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) goto epilogue_done;
      tc_fence_after();
      const int64_t row = t.row0 + row_in_tile;
      const bool row_ok = row < t.row_end;
      const int64_t col0 = static_cast<int64_t>(t.n_tile) * BN + g * CPW;
      const uint32_t acc_addr = lane_addr + static_cast<uint32_t>(tb * BN + g * CPW);
      if (p.splits == 1 && t.tail_slot < 0 && !p.out_f32) {
        // Read all of this warp's columns as packed bf16 first and hand the
        // accumulator back, so the next tile's MMAs start before the stores.
        uint32_t h[NCH][16];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(acc_addr + 32 * c, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]),
                                                      __uint_as_float(v[2 * j + 1]));
            h[c][j] = *reinterpret_cast<uint32_t*>(&b2);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
        const int64_t slab0 = t.row0 + quad * 32;
        if (p.y_tma && slab0 < t.row_end && (!GROUPED || slab0 + 32 <= t.row_end)) {
          // Staged TMA stores; rows past M and columns past N are clipped.
          uint8_t* box = out_boxes + e * kOutBoxBytes;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            if (col0 + 32 * c >= p.N) break;
            store_out_box(&tmap_y, box, lane, h[c], static_cast<int32_t>(col0 + 32 * c),
                          static_cast<int32_t>(slab0));
          }
        } else if (row_ok) {
          __nv_bfloat16* yrow = p.y + row * p.N;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const int64_t col = col0 + 32 * c;
            if (vec_store && col + 32 <= p.N) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(yrow + col + 8 * q) =
                    make_uint4(h[c][4 * q], h[c][4 * q + 1], h[c][4 * q + 2], h[c][4 * q + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const uint32_t pair = h[c][j >> 1];
                const uint16_t bits = static_cast<uint16_t>((j & 1) ? (pair >> 16) : (pair & 0xFFFFu));
                if (col + j < p.N) yrow[col + j] = __ushort_as_bfloat16(bits);
              }
            }
          }
        }
      } else {
        // FP32 split-K partials, chunk by chunk: staged TMA stores into split
        // t.split of the workspace (rows past M clipped), else direct stores.
        const int64_t slab0 = t.row0 + quad * 32;
        const bool slab_tma = p.y_tma == 2 && slab0 < t.row_end;
        uint8_t* box = out_boxes + e * kOutBoxBytes;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(acc_addr + 32 * c, v);
          tmem_ld_wait(v);
          if (c + 1 == NCH) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[tb]);
          }
          const int64_t col = col0 + 32 * c;
          if (!GROUPED && t.tail_slot >= 0) {
            // FP32 partial of a split tail unit: the whole 128 x BN tile
            // (rows and columns past the matrix are masked by the reduction).
            float* dst = p.tail_ws + (static_cast<int64_t>(t.tail_slot) * BM + row_in_tile) * BN +
                         g * CPW + 32 * c;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(dst + 4 * q) =
                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                              __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
            continue;
          }
          if (slab_tma) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (col + 16 * hh >= p.N) break;
              uint32_t w16[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) w16[j] = v[16 * hh + j];
              store_out_box(&tmap_y, box, lane, w16, static_cast<int32_t>(col + 16 * hh),
                            static_cast<int32_t>(slab0), t.split);
            }
            continue;
          }
          if (!row_ok) continue;
          float* wrow = p.ws + (static_cast<int64_t>(t.split) * p.M + row) * p.N;
          if ((p.N % 4) == 0 && col + 32 <= p.N) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(wrow + col + 4 * q) =
                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                              __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col + j < p.N) wrow[col + j] = __uint_as_float(v[j]);
          }
        }
      }
      if (++tb == C::kAccBufs) {
        tb = 0;
        tphase ^= 1u;
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

}  // namespace gemm
}  // namespace fp8bs
