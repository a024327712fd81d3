// Host-side check of the grouped GEMM's unit decoding (gemm::grouped_unit,
// the __host__ __device__ function the kernel calls) over the group table the
// kernel builds in shared memory: tile_prefix[g] (g <= G) = m tiles of the
// groups before g, and row_off[g] = tile_prefix[kMaxGroups + 1 + g] = device
// offset g clamped to [0, M]; group g owns rows [row_off[g],
// max(row_off[g + 1], row_off[g])).  For many group layouts (empty groups,
// offsets past M) every row of every group must be computed exactly once per
// n tile, over all K blocks, and no row outside the groups at all.  Offsets
// outside the contract (negative, decreasing) may make clamped groups overlap;
// for them every unit must still stay inside its group's clamped rows and
// inside [0, M).  Built and run on the CPU by
// tests/test_grouped_schedule.py; prints "ok ..." or the first failure.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "gemm.cuh"

namespace {

using fp8bs::gemm::kMaxGroups;

uint64_t g_state = 0x2545F4914F6CDD1Dull;
uint32_t rnd() {
  g_state ^= g_state << 13;
  g_state ^= g_state >> 7;
  g_state ^= g_state << 17;
  return static_cast<uint32_t>(g_state >> 32);
}

bool check(const std::vector<int64_t>& offsets, int64_t M, int n_tiles, int kbn, bool in_contract,
           long* rows_checked) {
  const int G = static_cast<int>(offsets.size()) - 1;
  std::vector<int> table(2 * (kMaxGroups + 1), 0);
  int* row_off = table.data() + kMaxGroups + 1;
  for (int g = 0; g <= G; ++g) {
    const int64_t o = offsets[g] < 0 ? 0 : (offsets[g] > M ? M : offsets[g]);
    row_off[g] = static_cast<int>(o);
  }
  int carry = 0;
  for (int g = 0; g < G; ++g) {
    const int lo = row_off[g], hi = row_off[g + 1] > lo ? row_off[g + 1] : lo;
    table[g] = carry;
    carry += (hi - lo + 127) / 128;
  }
  table[G] = carry;
  const int num_units = carry * n_tiles;

  fp8bs::gemm::Params p{};
  p.M = M;
  p.n_tiles = n_tiles;
  p.kbn = kbn;
  p.groups = G;
  // owner[row] = group that owns the row, or -1
  std::vector<int> owner(static_cast<size_t>(M), -1);
  for (int g = 0; g < G; ++g) {
    const int lo = row_off[g], hi = row_off[g + 1] > lo ? row_off[g + 1] : lo;
    for (int r = lo; r < hi; ++r) owner[r] = g;
  }
  std::vector<unsigned char> cov(static_cast<size_t>(M) * n_tiles, 0);
  for (int u = 0; u < num_units; ++u) {
    const fp8bs::gemm::Unit t = fp8bs::gemm::grouped_unit<128>(p, table.data(), u);
    const int lo = row_off[t.group], hi = row_off[t.group + 1] > lo ? row_off[t.group + 1] : lo;
    if (t.group < 0 || t.group >= G || t.n_tile < 0 || t.n_tile >= n_tiles || t.kb0 != 0 ||
        t.kb1 != kbn || t.row0 < lo || t.row0 >= hi || t.row_end != hi ||
        (t.row0 - lo) % 128 != 0) {
      std::printf("G=%d M=%lld unit %d -> group %d rows [%lld, %lld) n %d K [%d, %d)\n", G,
                  (long long)M, u, t.group, (long long)t.row0, (long long)t.row_end, t.n_tile,
                  t.kb0, t.kb1);
      return false;
    }
    const int64_t end = t.row0 + 128 < t.row_end ? t.row0 + 128 : t.row_end;
    for (int64_t r = t.row0; r < end; ++r) {
      if (r < 0 || r >= M) {
        std::printf("G=%d M=%lld: unit %d reaches row %lld\n", G, (long long)M, u, (long long)r);
        return false;
      }
      unsigned char& c = cov[static_cast<size_t>(r) * n_tiles + t.n_tile];
      if (c++ && in_contract) {
        std::printf("G=%d M=%lld: row %lld n tile %d computed twice\n", G, (long long)M,
                    (long long)r, t.n_tile);
        return false;
      }
    }
  }
  if (!in_contract) {
    *rows_checked += M * n_tiles;
    return true;
  }
  for (int64_t r = 0; r < M; ++r)
    for (int n = 0; n < n_tiles; ++n) {
      // clamped non-decreasing ranges: a row belongs to at most one group
      const bool want = owner[r] >= 0;
      if (cov[static_cast<size_t>(r) * n_tiles + n] != (want ? 1 : 0)) {
        std::printf("G=%d M=%lld: row %lld n tile %d computed %d times, owner %d\n", G,
                    (long long)M, (long long)r, n, cov[static_cast<size_t>(r) * n_tiles + n],
                    owner[r]);
        return false;
      }
    }
  *rows_checked += M * n_tiles;
  return true;
}

}  // namespace

int main() {
  long cases = 0, rows = 0;
  const int gs[] = {1, 2, 3, 7, 32, 33, 256, 1024};
  const int ns[] = {1, 3, 8};
  for (int G : gs)
    for (int n_tiles : ns)
      for (int rep = 0; rep < 6; ++rep) {
        std::vector<int64_t> off(G + 1, 0);
        const int mode = rep % 3;
        for (int g = 1; g <= G; ++g) {
          const int64_t cnt = (rnd() % 4 == 0) ? 0 : static_cast<int64_t>(rnd() % (mode == 2 ? 700 : 300));
          off[g] = off[g - 1] + cnt;
        }
        int64_t M = off[G];
        if (mode == 1) M = M - M / 3;   // offsets past M: the tail groups are clipped
        if (mode == 2 && G > 2) {       // out-of-contract offsets the kernel clamps
          off[1] = -50;
          off[G / 2] = off[G / 2 - 1] - 7;
        }
        if (M <= 0) M = 1;
        if (!check(off, M, n_tiles, 1 + static_cast<int>(rnd() % 56), mode != 2, &rows)) return 1;
        ++cases;
      }
  std::printf("ok %ld group layouts, %ld (row, n tile) pairs\n", cases, rows);
  return 0;
}
