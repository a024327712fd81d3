// Host-side check of the GEMM's dense tile order (gemm::tile_mn, the same
// __host__ __device__ function the kernels use): for every shape below, the
// tile indices 0 .. m_tiles * n_tiles - 1 map one to one onto (m tile, n tile)
// pairs in range, and inside a band the m tile changes slowest.  The same for
// the transposing kernels' tile order (fp8bs::tile_coords).  Built and run on
// the CPU by tests/test_tile_order.py; prints "ok" or the first failure.
#include <cstdio>
#include <vector>

#include "gemm.cuh"
#include "transpose.cuh"

int main() {
  const int ms[] = {1, 2, 3, 7, 32, 144, 513};
  const int ns[] = {1, 2, 5, 8, 28, 72, 144};
  long cases = 0;
  for (int mt : ms)
    for (int nt : ns)
      for (int g = 1; g <= nt; g += (g < 8 ? 1 : 7)) {
        std::vector<int> seen(static_cast<size_t>(mt) * nt, 0);
        int prev_m = -1, prev_n = -1;
        for (int tile = 0; tile < mt * nt; ++tile) {
          int m = -1, n = -1;
          fp8bs::gemm::tile_mn(tile, mt, nt, g, m, n);
          if (m < 0 || m >= mt || n < 0 || n >= nt) {
            std::printf("out of range: mt=%d nt=%d g=%d tile=%d -> (%d, %d)\n", mt, nt, g, tile, m, n);
            return 1;
          }
          if (seen[static_cast<size_t>(m) * nt + n]++) {
            std::printf("repeat: mt=%d nt=%d g=%d tile=%d -> (%d, %d)\n", mt, nt, g, tile, m, n);
            return 1;
          }
          // consecutive tiles inside one band: same m tile, or the next one
          if (tile > 0 && n / g == prev_n / g && m != prev_m && m != prev_m + 1) {
            std::printf("order: mt=%d nt=%d g=%d tile=%d\n", mt, nt, g, tile);
            return 1;
          }
          prev_m = m;
          prev_n = n;
          ++cases;
        }
      }
  // The transposing kernels' tile order (fp8bs::tile_coords): tiles
  // 0 .. bands * tiles_c - 1 map one to one onto (row band, column tile)
  // pairs, and inside a group of kBandGroup bands the band changes fastest.
  const int64_t bands_list[] = {1, 2, 7, 8, 9, 16, 17, 32, 56, 144};
  const int64_t cols_list[] = {1, 2, 3, 8, 32, 56, 144};
  for (int64_t bands : bands_list)
    for (int64_t tc_n : cols_list) {
      std::vector<int> seen(static_cast<size_t>(bands * tc_n), 0);
      int64_t prev_r = -1, prev_c = -1;
      for (int64_t tile = 0; tile < bands * tc_n; ++tile) {
        int64_t tr = -1, tc = -1;
        fp8bs::tile_coords(tile, bands, tc_n, tr, tc);
        if (tr < 0 || tr >= bands || tc < 0 || tc >= tc_n) {
          std::printf("transpose tile out of range: bands=%lld cols=%lld tile=%lld -> (%lld, %lld)\n",
                      (long long)bands, (long long)tc_n, (long long)tile, (long long)tr, (long long)tc);
          return 1;
        }
        if (seen[static_cast<size_t>(tr * tc_n + tc)]++) {
          std::printf("transpose tile repeat: bands=%lld cols=%lld tile=%lld\n", (long long)bands,
                      (long long)tc_n, (long long)tile);
          return 1;
        }
        // the band advances first, within its group of kBandGroup bands
        if (tile > 0 && tr / fp8bs::kBandGroup == prev_r / fp8bs::kBandGroup && tc == prev_c &&
            tr != prev_r + 1) {
          std::printf("transpose order: bands=%lld cols=%lld tile=%lld\n", (long long)bands,
                      (long long)tc_n, (long long)tile);
          return 1;
        }
        prev_r = tr;
        prev_c = tc;
        ++cases;
      }
    }
  std::printf("ok %ld\n", cases);
  return 0;
}
