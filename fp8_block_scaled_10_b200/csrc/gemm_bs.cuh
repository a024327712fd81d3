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
// Scale factors in TMEM: for every 128 rows and one 128-wide K block, a
// 512-byte atom whose byte 16*(r%32) + 4*(r/32) + j holds the exponent of row
// r for the j-th 32-wide K sub-block (all four equal here: one scale per 128
// K elements), copied from shared memory by tcgen05.cp 32x128b.warpx4 into
// 4 TMEM columns.  The MMA for sub-block j selects byte j.
//
// Roles (persistent, one CTA per SM, 12 warps):
//   warp 0      TMA producer of A [128 x 128] and W [BN x 128] tiles.
//   warp 1      TMEM owner; one lane copies each stage's scale atoms into a
//               TMEM ring and issues the block-scaled MMAs.
//   warp 2      scale producer: reads a_s / w_s (prefetched four K blocks
//               ahead), writes the exponent atoms into the stage's shared
//               memory and checks that each scale is a positive normal power
//               of two (else device error FP8BS_ERR_SCALE = 6).
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
  static constexpr int kSFBytes = 512 * kSFAtoms;
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kAccBufs = (BN == 256) ? 1 : 2;    // TMEM accumulators
  static constexpr int kSFCols = 4 * kSFAtoms;            // TMEM columns per stage
  static constexpr int kSFBase = kAccBufs * BN;
  static constexpr int kTmemCols = 512;
  static_assert(kSFBase + kStages * kSFCols <= kTmemCols, "TMEM budget");
  static constexpr int kEpiWarps = 8;
  static constexpr int kColsPerWarp = BN / 2;
  static constexpr int kFirstEpiWarp = 4;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr int kCtrlBytes = 256;
  static constexpr int kGroupBytes = 4 * kGroupTableInts;
  __host__ __device__ static constexpr int out_offset(bool grouped) {
    return (kStages * (kStageBytes + kSFBytes) + kCtrlBytes + (grouped ? kGroupBytes : 0) + 1023) &
           ~1023;
  }
  __host__ __device__ static constexpr int smem_bytes(bool grouped) {
    return out_offset(grouped) + kEpiWarps * kOutBoxBytes + 1024;
  }
};

template <int kStages>
struct BsCtrl {
  uint64_t full[kStages];    // TMA bytes + the scale producer's arrival
  uint64_t empty[kStages];
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
      reinterpret_cast<BsCtrl<C::kStages>*>(sf_tiles + C::kStages * C::kSFBytes);
  static_assert(sizeof(BsCtrl<C::kStages>) <= C::kCtrlBytes, "control block too large");
  uint64_t* full = ctrl->full;
  uint64_t* empty = ctrl->empty;
  uint64_t* tfull = ctrl->tfull;
  uint64_t* tempty = ctrl->tempty;
  uint64_t* flush = &ctrl->flush;
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
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
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
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      for (int u = unit_start; u < num_units; u += unit_step) {
        const Unit t = unit_of(u);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) goto producer_done;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_2d(a_tiles + stage * C::kABytes, &tmap_a, &full[stage], kb * BK,
                      static_cast<int32_t>(t.row0));
          tma_load_2d(b_tiles + stage * C::kBBytes, &tmap_w, &full[stage], kb * BK,
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
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale producer
    // Walks the same (unit, K block) sequence as the TMA producer; a second
    // cursor runs four steps ahead and loads the scales into a ring of
    // registers, so the loads of step i+4 overlap the atoms of step i.
    // W values per lane and step: one block scale per 128-row atom, or with
    // BROW the lane's four rows of each atom.
    constexpr int kWVals = BROW ? BN / 32 : BN / 128;
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
    auto load = [&](const Cursor& c, float (&va)[4], float (&vw)[kWVals]) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t row = c.row0 + lane + 32 * j;
        va[j] = (c.valid && row < c.row_end)
                    ? __ldg(BROW ? p.sa + c.kb * p.M + row : p.sa + row * p.kbn + c.kb)
                    : 1.0f;
      }
      if (BROW) {
        // value 4a + j: row 128a + lane + 32j of the tile's W rows, from the
        // K-block-major table sw [kbn][N] (coalesced across lanes)
#pragma unroll
        for (int i = 0; i < kWVals; ++i) {
          const int64_t n = c.n0 + 128 * (i / 4) + lane + 32 * (i % 4);
          vw[i] = (c.valid && n < p.N) ? __ldg(p.sw + c.kb * static_cast<int64_t>(p.N) + n) : 1.0f;
        }
      } else {
#pragma unroll
        for (int a = 0; a < BN / 128; ++a) {
          const int nb = c.nb0 + a;
          vw[a] = (c.valid && nb < p.nbn)
                      ? __ldg(p.sw + (static_cast<int64_t>(c.group) * p.nbn + nb) * p.kbn + c.kb)
                      : 1.0f;
        }
      }
    };
    float ra[4][4], rw[4][kWVals];
    Cursor ahead, cur;
    begin(ahead, unit_start);
    begin(cur, unit_start);
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      load(ahead, ra[d], rw[d]);
      next(ahead);
    }
    int stage = 0;
    uint32_t phase = 0;
    bool bad = false;
    while (cur.valid) {
#pragma unroll
      for (int ph = 0; ph < 4; ++ph) {
        if (!cur.valid) break;
        const bool ok = mbar_wait(&empty[stage], phase ^ 1u, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok)) goto scales_done;
        uint8_t* atoms = sf_tiles + stage * C::kSFBytes;
        uint4 v;
        v.x = ue8m0_byte(ra[ph][0], &bad) * 0x01010101u;
        v.y = ue8m0_byte(ra[ph][1], &bad) * 0x01010101u;
        v.z = ue8m0_byte(ra[ph][2], &bad) * 0x01010101u;
        v.w = ue8m0_byte(ra[ph][3], &bad) * 0x01010101u;
        *reinterpret_cast<uint4*>(atoms + 16 * lane) = v;
#pragma unroll
        for (int a = 0; a < BN / 128; ++a) {
          if (BROW) {
            uint4 w;
            w.x = ue8m0_byte(rw[ph][4 * a + 0], &bad) * 0x01010101u;
            w.y = ue8m0_byte(rw[ph][4 * a + 1], &bad) * 0x01010101u;
            w.z = ue8m0_byte(rw[ph][4 * a + 2], &bad) * 0x01010101u;
            w.w = ue8m0_byte(rw[ph][4 * a + 3], &bad) * 0x01010101u;
            *reinterpret_cast<uint4*>(atoms + 512 * (1 + a) + 16 * lane) = w;
          } else {
            const uint32_t e = ue8m0_byte(rw[ph][a], &bad) * 0x01010101u;
            *reinterpret_cast<uint4*>(atoms + 512 * (1 + a) + 16 * lane) = make_uint4(e, e, e, e);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        load(ahead, ra[ph], rw[ph]);
        next(ahead);
        next(cur);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  scales_done:
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report_error(6);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_block_scaled(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int tb = 0;
      uint32_t tphase = 0;
      for (int u = unit_start; u < num_units; u += unit_step) {
        const Unit t = unit_of(u);
        // The epilogue has drained this accumulator (tile u - 2 * step).
        if (!mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag)) goto mma_done;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * BN);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) goto mma_done;
          tc_fence_after();
          // Scale atoms of this stage into its TMEM slot (A, then W).
          const uint32_t tsf = tmem_base + static_cast<uint32_t>(C::kSFBase + stage * C::kSFCols);
          const uint8_t* atoms = sf_tiles + stage * C::kSFBytes;
#pragma unroll
          for (int a = 0; a < C::kSFAtoms; ++a)
            tmem_copy_32x128b_x4(tsf + 4 * a, smem_desc_rows16(smem_addr(atoms + 512 * a)));
          const uint32_t a_addr = smem_addr(a_tiles + stage * C::kABytes);
          const uint32_t b_addr = smem_addr(b_tiles + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint32_t sub = static_cast<uint32_t>(k);
            mma_mxf8_block_scaled(d_tmem, smem_desc_k_sw128(a_addr + 32 * k),
                                  smem_desc_k_sw128(b_addr + 32 * k),
                                  idesc | (sub << 29) | (sub << 4), tsf | (sub << 30),
                                  (tsf + 4) | (sub << 30), (kb > t.kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        mma_commit(&tfull[tb]);
        if (++tb == C::kAccBufs) {
          tb = 0;
          tphase ^= 1u;
        }
      }
    mma_done:
      mma_commit(flush);
      mbar_wait(flush, 0, nullptr);
    }
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
