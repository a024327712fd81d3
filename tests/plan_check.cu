// Host-side check of the dense GEMM plans (plan.h) against the kernels' own
// unit decoding (gemm::dense_unit, the __host__ __device__ function both GEMM
// kernels call).  For many shapes, SM counts and both kernels:
//   - the plan's fields are consistent (tile grid, K split, split tail, grid,
//     band width, workspace);
//   - the work units 0 .. units-1, decoded as the kernels decode them, cover
//     every (m tile, n tile, K block) exactly once, and every split-tail unit
//     writes its own partial slot, the one the tail reduction reads for that
//     tile.
// Then the plans recorded on a 148-SM B200 for the benchmark shapes.
// Built and run on the CPU by tests/test_gemm_plan.py; prints "ok ..." or the
// first failure.
#include <cstdio>
#include <cstring>
#include <vector>

#include "plan.h"

using fp8bs::GemmKind;
using fp8bs::Plan;

namespace {

const char* kind_name(GemmKind k) {
  return k == GemmKind::kPromotion ? "promotion" : (k == GemmKind::kBlockScaled ? "block-scaled" : "row-scaled");
}

#define FAIL(...)                                                                         \
  do {                                                                                    \
    std::printf("M=%lld N=%lld K=%lld sms=%d %s: ", (long long)M, (long long)N,          \
                (long long)K, sms, kind_name(kind));                                      \
    std::printf(__VA_ARGS__);                                                             \
    std::printf("\n");                                                                    \
    return false;                                                                         \
  } while (0)

bool check(int64_t M, int64_t N, int64_t K, int sms, GemmKind kind, long* cells) {
  const Plan pl = fp8bs::plan_gemm(M, N, K, sms, kind);
  fp8bs::gemm::Params p{};
  fp8bs::set_schedule(p, pl, M, N, K);
  const int kbn = static_cast<int>(K / 128);
  const bool tail = pl.tail_splits > 0;

  if (pl.bn != 256 && pl.bn != 192 && pl.bn != 128) FAIL("bn=%d", pl.bn);
  if (pl.bn == 192 && (kind != GemmKind::kPromotion || M <= 128)) FAIL("192-wide tile planned");
  if (pl.m_tiles != (M + 127) / 128 || pl.n_tiles != (N + pl.bn - 1) / pl.bn)
    FAIL("tile grid %d x %d", pl.m_tiles, pl.n_tiles);
  const int64_t tiles = static_cast<int64_t>(pl.m_tiles) * pl.n_tiles;
  if (pl.splits < 1 || pl.kb_per_split < 1 || (pl.splits - 1) * pl.kb_per_split >= kbn ||
      pl.splits * pl.kb_per_split < kbn)
    FAIL("K split %d x %d for %d K blocks", pl.splits, pl.kb_per_split, kbn);
  if (pl.splits > 1 && tiles >= sms) FAIL("K split although %lld tiles fill %d SMs", (long long)tiles, sms);
  if (tail) {
    if (pl.splits != 1) FAIL("split tail on a K split");
    if (pl.tail_tiles <= 0 || 2 * pl.tail_tiles > sms || pl.full_units != tiles - pl.tail_tiles ||
        pl.full_units % sms != 0)
      FAIL("tail of %d tiles after %d full units", pl.tail_tiles, pl.full_units);
    if (pl.tail_splits < 2 || (pl.tail_splits - 1) * pl.tail_kbps >= kbn ||
        pl.tail_splits * pl.tail_kbps < kbn)
      FAIL("tail split %d x %d", pl.tail_splits, pl.tail_kbps);
    if (pl.units != pl.full_units + pl.tail_tiles * pl.tail_splits) FAIL("units %d", pl.units);
    if (fp8bs::plan_workspace(pl, M, N) > fp8bs::kTailWorkspaceCap) FAIL("tail workspace");
  } else if (pl.units != tiles * pl.splits) {
    FAIL("units %d for %lld tiles x %d splits", pl.units, (long long)tiles, pl.splits);
  }
  if (pl.grid < 1 || pl.grid > sms || pl.grid > pl.units) FAIL("grid %d", pl.grid);
  if (pl.n_group < 1 || pl.n_group > pl.n_tiles) FAIL("n_group %d", pl.n_group);
  if (pl.n_group != 1 && (pl.splits > 1 || M <= 128)) FAIL("band order with n_group %d", pl.n_group);

  std::vector<unsigned char> cov(static_cast<size_t>(tiles) * kbn, 0);
  std::vector<unsigned char> slot(tail ? static_cast<size_t>(pl.tail_tiles) * pl.tail_splits : 0, 0);
  for (int u = 0; u < pl.units; ++u) {
    const fp8bs::gemm::Unit t = fp8bs::gemm::dense_unit<128>(p, u);
    const int64_t m_tile = t.row0 / 128;
    if (t.row0 % 128 != 0 || m_tile < 0 || m_tile >= pl.m_tiles || t.n_tile < 0 ||
        t.n_tile >= pl.n_tiles || t.row_end != M)
      FAIL("unit %d -> rows %lld, n tile %d", u, (long long)t.row0, t.n_tile);
    if (t.kb0 < 0 || t.kb0 >= t.kb1 || t.kb1 > kbn) FAIL("unit %d -> K blocks [%d, %d)", u, t.kb0, t.kb1);
    if (t.tail_slot >= 0) {
      if (!tail || t.tail_slot >= static_cast<int>(slot.size()) || slot[t.tail_slot]++)
        FAIL("unit %d -> tail slot %d", u, t.tail_slot);
      // The reduction sums slots tt * tail_splits + s into tile full_units + tt.
      const int tt = t.tail_slot / pl.tail_splits;
      int rm = -1, rn = -1;
      fp8bs::gemm::tile_mn(pl.full_units + tt, pl.m_tiles, pl.n_tiles, pl.n_group, rm, rn);
      if (rm != m_tile || rn != t.n_tile || t.split != t.tail_slot % pl.tail_splits)
        FAIL("unit %d: tail slot %d belongs to tile (%d, %d), unit computes (%lld, %d)", u,
             t.tail_slot, rm, rn, (long long)m_tile, t.n_tile);
    } else if (tail && u >= pl.full_units) {
      FAIL("tail unit %d without a slot", u);
    }
    if (t.split < 0 || t.split >= (tail && t.tail_slot >= 0 ? pl.tail_splits : pl.splits))
      FAIL("unit %d -> split %d", u, t.split);
    for (int kb = t.kb0; kb < t.kb1; ++kb) {
      unsigned char& c = cov[(static_cast<size_t>(m_tile) * pl.n_tiles + t.n_tile) * kbn + kb];
      if (c++) FAIL("unit %d repeats tile (%lld, %d) K block %d", u, (long long)m_tile, t.n_tile, kb);
    }
  }
  for (size_t i = 0; i < cov.size(); ++i)
    if (!cov[i]) FAIL("tile %zu K block %zu never computed", i / kbn, i % kbn);
  *cells += static_cast<long>(cov.size());
  return true;
}

struct Recorded {
  int64_t M, N, K;
  GemmKind kind;
  int bn, splits, kb_per_split, units, grid, tail_tiles, tail_splits, n_group;
};

}  // namespace

int main() {
  const int64_t ms[] = {1, 8, 33, 64, 100, 128, 129, 300, 1000, 1200, 4096, 18432};
  const int64_t ns[] = {128, 130, 576, 2048, 4000, 7168, 18432};
  const int64_t ks[] = {128, 256, 1024, 4096, 7168, 18432};
  const int sm_counts[] = {148, 132, 20};
  const GemmKind kinds[] = {GemmKind::kPromotion, GemmKind::kBlockScaled, GemmKind::kRowScaled};
  long cases = 0, cells = 0;
  for (int64_t M : ms)
    for (int64_t N : ns)
      for (int64_t K : ks)
        for (int sms : sm_counts)
          for (GemmKind kind : kinds) {
            if (!check(M, N, K, sms, kind, &cells)) return 1;
            ++cases;
          }

  // Plans the library reported (fp8bs_gemm_plan_string) on a 148-SM B200 for
  // the benchmark's shapes; the block-scaled entry plans the same ones.
  const Recorded rec[] = {
      {4096, 18432, 7168, GemmKind::kPromotion, 256, 1, 56, 2304, 148, 0, 0, 1},
      {4096, 18432, 7168, GemmKind::kBlockScaled, 256, 1, 56, 2304, 148, 0, 0, 1},
      {4096, 7168, 18432, GemmKind::kPromotion, 256, 1, 144, 1016, 148, 8, 16, 4},
      {4096, 7168, 18432, GemmKind::kBlockScaled, 256, 1, 144, 1016, 148, 8, 16, 4},
      {4096, 576, 7168, GemmKind::kPromotion, 128, 1, 56, 292, 148, 12, 12, 1},
      {1, 18432, 7168, GemmKind::kPromotion, 128, 1, 56, 144, 144, 0, 0, 1},
      {64, 18432, 7168, GemmKind::kPromotion, 128, 1, 56, 144, 144, 0, 0, 1},
      {1, 7168, 18432, GemmKind::kPromotion, 256, 5, 29, 140, 140, 0, 0, 1},
      {64, 7168, 18432, GemmKind::kPromotion, 256, 5, 29, 140, 140, 0, 0, 1},
  };
  for (const Recorded& r : rec) {
    const Plan pl = fp8bs::plan_gemm(r.M, r.N, r.K, 148, r.kind);
    if (pl.bn != r.bn || pl.splits != r.splits || pl.kb_per_split != r.kb_per_split ||
        pl.units != r.units || pl.grid != r.grid || pl.tail_tiles != r.tail_tiles ||
        pl.tail_splits != r.tail_splits || pl.n_group != r.n_group) {
      std::printf("recorded plan changed: M=%lld N=%lld K=%lld %s: bn=%d splits=%d kbps=%d units=%d "
                  "grid=%d tail=%d x %d n_group=%d\n",
                  (long long)r.M, (long long)r.N, (long long)r.K, kind_name(r.kind), pl.bn,
                  pl.splits, pl.kb_per_split, pl.units, pl.grid, pl.tail_tiles, pl.tail_splits,
                  pl.n_group);
      return 1;
    }
  }
  std::printf("ok %ld plans, %ld (tile, K block) cells\n", cases, cells);
  return 0;
}
