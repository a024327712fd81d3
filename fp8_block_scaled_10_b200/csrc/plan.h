// GEMM planning for the dense FP8 GEMM kernels (gemm.cuh, gemm_bs.cuh): the
// tile width BN, the K split, the split tail and the band width of the tile
// order, chosen from the problem size and the SM count, and the copy of a
// plan into the kernels' parameters.  Host code only; the C ABI (fp8bs.cu)
// plans every dense launch here, and a host build checks the plans against
// the kernels' own unit decoding (gemm::dense_unit) without a GPU.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>

#include "fp8bs.h"
#include "gemm.cuh"

namespace fp8bs {

struct Plan {
  int bn;
  int m_tiles, n_tiles;
  int splits, kb_per_split;
  int units;
  int grid;   // persistent CTAs
  // Split tail (see gemm::Params): 0 = none.
  int full_units = 0, tail_tiles = 0, tail_splits = 0, tail_kbps = 0;
  int n_group = 1;   // band width of the tile order (gemm::tile_mn)
  double est_us = 0.0;   // the planner's time estimate (prefill-sized M)
};

// Band width of the dense tile order for one K split.  m fastest (width 1)
// reads each W tile once and A once per n tile, from L2 when A fits there
// beside the W tiles in flight (up to kAResidentBytes).  A larger A would
// come from HBM once per n tile; a band of n tiles whose W fits in
// kWBandBytes of L2 then reads A once per band instead.  (Measured on B200:
// the weight-gradient shape M = 18432, N = 7168, K = 4096 read 1.7 GB per
// launch m-fastest, against 0.64 GB of operands and output.)
constexpr int64_t kAResidentBytes = 40ll << 20;
constexpr int64_t kWBandBytes = 20ll << 20;
inline int choose_n_group(int64_t M, int64_t K, int bn, int n_tiles) {
  if (M * K <= kAResidentBytes) return 1;
  const int64_t g = kWBandBytes / (static_cast<int64_t>(bn) * K);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g, n_tiles)));
}

// The split tail's FP32 partials are kept within this many bytes, so that
// every prefill plan also fits the library's static scratch array.
constexpr size_t kTailWorkspaceCap = FP8BS_STATIC_SCRATCH_BYTES;

inline double wave_efficiency(int64_t units, int slots) {
  const int64_t waves = (units + slots - 1) / slots;
  return static_cast<double>(units) / static_cast<double>(waves * slots);
}

// The two GEMM kernels the planner serves.
// kRowScaled: the promotion kernel with one scale per row of W (per column of
// y) and K block, whose epilogue multiplies each column's scale in.
enum class GemmKind { kPromotion, kBlockScaled, kRowScaled };

// Time per K block of one 128-row work unit, in microseconds, measured on
// B200 at M = 4096 with every SM busy.
//   promotion kernel: 128 x 256 tile ~0.55, 128 x 192 ~0.48, 128 x 128
//     ~0.36 (the tensor core and the epilogue's FP32 promotion overlap; the
//     wider tile moves fewer operand bytes per FLOP);
//   block-scaled kernel: 128 x 256 ~0.5, 128 x 128 ~1/3 (operand feed).
inline double kb_time_us(GemmKind kind, int bn) {
  if (kind == GemmKind::kPromotion) return bn == 256 ? 0.55 : (bn == 192 ? 0.48 : 0.36);
  if (kind == GemmKind::kRowScaled) return bn == 256 ? 0.62 : 0.40;
  return bn == 256 ? 0.5 : 1.0 / 3.0;
}

// Chooses tile width and K split.
//
// M > 128 (several 128-row tiles share each W tile): the estimated time is
// waves of work units x K blocks per unit x kb_time_us, plus, for a K split,
// the FP32 partials' round trip through HBM and the reduction launch.  When
// the tiles fill the GPU but their last wave would keep at most half of the
// SMs busy, the plan can split only the tiles of that wave along
// K ("split tail", both kernels): the whole waves run unchanged and the
// tail's partials, a few MB, are summed by a small reduction.
//
// M <= 128 (decode): the weight stream from HBM bounds every tile width
// alike; the score is the fraction of persistent slots kept busy, with a
// small cost per split, preferring wider tiles.
inline Plan plan_gemm(int64_t M, int64_t N, int64_t K, int sms,
                      GemmKind kind = GemmKind::kPromotion) {
  Plan best{};
  double best_score = -1.0;
  double best_time = 1e30;
  const int kbn = static_cast<int>(K / 128);
  const bool compute_bound = M > 128;
  const int slots = sms;
  for (int bn : {256, 192, 128}) {
    if (bn == 192 && (kind != GemmKind::kPromotion || !compute_bound)) continue;
    const int m_tiles = static_cast<int>((M + 127) / 128);
    const int n_tiles = static_cast<int>((N + bn - 1) / bn);
    const int64_t tiles = static_cast<int64_t>(m_tiles) * n_tiles;
    // Split K only when the tiles alone cannot fill the GPU.
    const int max_split = tiles >= slots ? 1 : std::min(16, std::max(1, kbn / 4));
    for (int s = 1; s <= max_split; ++s) {
      const int per = (kbn + s - 1) / s;
      const int splits = (kbn + per - 1) / per;
      if (splits != s) continue;
      const int64_t units = tiles * splits;
      bool better;
      Plan cand{bn, m_tiles, n_tiles, splits, per, static_cast<int>(units),
                static_cast<int>(std::min<int64_t>(units, slots))};
      if (compute_bound) {
        const double kb_us = kb_time_us(kind, bn);
        const double waves = static_cast<double>((units + slots - 1) / slots);
        double t = waves * per * kb_us;
        if (splits > 1)   // partials written and read back (HBM ~5 TB/s), bf16 out, launch
          t += (8.0 * splits + 2.0) * static_cast<double>(M) * N / 5.0e6 + 5.0;
        const int64_t tail = tiles % slots;
        if (splits == 1 && tiles > slots && tail > 0 && 2 * tail <= slots) {
          const size_t tile_bytes = static_cast<size_t>(128) * bn * sizeof(float);
          const int64_t by_ws = static_cast<int64_t>(kTailWorkspaceCap / (tail * tile_bytes));
          const int ts = static_cast<int>(std::min<int64_t>({slots / tail, kbn / 4, by_ws}));
          if (ts >= 2) {
            const int tkb = (kbn + ts - 1) / ts;
            const double t_tail = static_cast<double>(tiles / slots) * per * kb_us +
                                  tkb * kb_us + 3.0;   // + the reduction launch
            if (t_tail < t) {
              t = t_tail;
              cand.full_units = static_cast<int>(tiles - tail);
              cand.tail_tiles = static_cast<int>(tail);
              cand.tail_splits = (kbn + tkb - 1) / tkb;
              cand.tail_kbps = tkb;
              cand.units = cand.full_units + cand.tail_tiles * cand.tail_splits;
              cand.grid = slots;
            }
          }
        }
        better = t < best_time - 1e-9;
        if (better) {
          best_time = t;
          cand.est_us = t;
        }
      } else {
        const double eff = wave_efficiency(units, slots);
        const double fill = static_cast<double>(std::min<int64_t>(M, 128)) / 128;
        const double feed = bn == 128 ? 0.97 : 1.0;
        const double split_cost = splits > 1 ? 0.95 - 0.002 * splits : 1.0;
        const double score = eff * feed * split_cost * (fill + 0.5 * (1 - fill));
        better = score > best_score + 1e-9;
        if (better) best_score = score;
      }
      if (better) best = cand;
    }
  }
  if (best.splits == 1 && compute_bound) best.n_group = choose_n_group(M, K, best.bn, best.n_tiles);
  return best;
}

// The fused linear layer (act_quant inside the GEMM launch, linear.cuh).
// When the GEMM's tiles leave SMs idle, those SMs quantize x instead: the
// launch has gemm_ctas CTAs walking the GEMM's tiles (one wave, no K split)
// and quant_ctas CTAs streaming x and writing q and s, each (m tile, K block)
// chunk announced by a ready flag that the GEMM CTAs wait for before they
// load it.
struct LinearPlan {
  bool fused = false;
  Plan gemm;            // the fused launch's tile plan (fused), else the GEMM's plan
  int gemm_ctas = 0;
  int quant_ctas = 0;
  double est_us = 0.0;
};

constexpr int kMinQuantCtas = 16;
// Measured on B200 (M = 4096, K = 7168, N = 576, 52 quantizer CTAs): a
// quantizer CTA moves ~35 GB/s (x read, q and s written; it is bound by its
// arithmetic, as act_quant is per SM), and a GEMM CTA spends ~0.64 us per K
// block on the round trip of reading its chunk's flag.  act_quant alone moves
// ~5.9 TB/s over all SMs.
constexpr double kQuantCtaGBs = 35.0;
constexpr double kFlagRoundTripUs = 0.64;
constexpr double kActQuantGBs = 5900.0;

inline size_t linear_flag_bytes(int64_t M, int64_t K) {
  return static_cast<size_t>((M + 127) / 128) * static_cast<size_t>(K / 128) * sizeof(int);
}

// The best fused launch for the shape (fused = false when none fits: the
// tiles must leave at least kMinQuantCtas SMs, and M must exceed 128).
inline LinearPlan plan_linear_fused(int64_t M, int64_t N, int64_t K, int sms) {
  LinearPlan lp;
  if (M <= 128) return lp;
  const double q_bytes = static_cast<double>(M) * K * 3.0 + 4.0 * M * (K / 128);
  const int kbn = static_cast<int>(K / 128);
  lp.est_us = 1e30;
  for (int bn : {256, 192, 128}) {
    const int m_tiles = static_cast<int>((M + 127) / 128);
    const int n_tiles = static_cast<int>((N + bn - 1) / bn);
    const int64_t tiles = static_cast<int64_t>(m_tiles) * n_tiles;
    if (tiles + kMinQuantCtas > sms) continue;
    const int q = sms - static_cast<int>(tiles);
    const double t = std::max(kbn * std::max(kb_time_us(GemmKind::kPromotion, bn), kFlagRoundTripUs),
                              q_bytes / (q * kQuantCtaGBs * 1e3)) + 2.0;
    if (t < lp.est_us - 1e-9) {
      Plan g{bn, m_tiles, n_tiles, 1, kbn, static_cast<int>(tiles), sms};
      g.est_us = t;
      lp.fused = true;
      lp.gemm = g;
      lp.gemm_ctas = static_cast<int>(tiles);
      lp.quant_ctas = q;
      lp.est_us = t;
    }
  }
  return lp;
}

// fp8_linear's choice: the fused launch when its estimate beats act_quant
// followed by the GEMM's own plan.
inline LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int sms) {
  LinearPlan lp;
  lp.gemm = plan_gemm(M, N, K, sms);
  const double q_bytes = static_cast<double>(M) * K * 3.0 + 4.0 * M * (K / 128);
  lp.est_us = (M > 128 ? lp.gemm.est_us : 0.0) + q_bytes / (kActQuantGBs * 1e3) + 2.0;
  const LinearPlan f = plan_linear_fused(M, N, K, sms);
  return (f.fused && f.est_us < lp.est_us - 1e-9) ? f : lp;
}

// Bytes of the K-block-major copies of the two scale tables that the
// row-scaled GEMM stages in its workspace.
inline size_t rowwise_stage_bytes(int64_t M, int64_t N, int64_t K) {
  return static_cast<size_t>(M + N) * static_cast<size_t>(K / 128) * sizeof(float);
}

inline size_t plan_workspace(const Plan& pl, int64_t M, int64_t N) {
  if (pl.tail_splits > 0)
    return static_cast<size_t>(pl.tail_tiles) * pl.tail_splits * 128 * pl.bn * sizeof(float);
  return pl.splits > 1 ? static_cast<size_t>(pl.splits) * M * N * sizeof(float) : 0;
}

// Copies the schedule of a plan into the kernel parameters: problem size,
// tile grid, tile order, K split and split tail.  Pointers, tensor maps and
// output modes are the caller's.
inline void set_schedule(gemm::Params& p, const Plan& pl, int64_t M, int64_t N, int64_t K) {
  p.M = M;
  p.N = static_cast<int>(N);
  p.kbn = static_cast<int>(K / 128);
  p.nbn = static_cast<int>((N + 127) / 128);
  p.m_tiles = pl.m_tiles;
  p.n_tiles = pl.n_tiles;
  p.n_group = pl.n_group;
  p.splits = pl.splits;
  p.kb_per_split = pl.kb_per_split;
  p.num_units = pl.units;
  p.full_units = pl.full_units;
  p.tail_tiles = pl.tail_tiles;
  p.tail_splits = pl.tail_splits;
  p.tail_kbps = pl.tail_kbps;
  p.groups = 1;
}

}  // namespace fp8bs
