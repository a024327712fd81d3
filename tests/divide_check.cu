// Host-side check of the division by an invariant divisor that the static
// quantizer and the dequantizer use for their row index (invariant_div on the
// host, div_invariant in the kernels; on the host div_invariant takes the high
// word of the 64-bit product, which __umulhi returns on the device).  For many
// divisors, every quotient at and around each sampled multiple of d, and at
// the ends of the 32-bit range, must equal n / d; for d = 7 every 32-bit n is
// checked.  Built and run on the CPU by tests/test_invariant_division.py;
// prints "ok ..." or the first failure.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "quant.cuh"

namespace {

bool check_one(uint32_t n, uint32_t d, const fp8bs::InvariantDiv& inv) {
  const uint32_t got = fp8bs::div_invariant(n, inv);
  if (got != n / d) {
    std::printf("d=%u n=%u: %u, expected %u\n", d, n, got, n / d);
    return false;
  }
  return true;
}

}  // namespace

int main() {
  std::vector<uint32_t> ds;
  for (uint32_t d = 1; d <= 4096; ++d) ds.push_back(d);
  for (int k = 12; k < 32; ++k) {
    const uint32_t p = 1u << k;
    ds.push_back(p - 1);
    ds.push_back(p);
    ds.push_back(p + 1);
  }
  for (uint32_t d : {224u, 448u, 1152u, 7168u, 18432u, 65535u, 1000003u, 2147483647u,
                     2147483649u, 4294967295u})
    ds.push_back(d);
  uint64_t state = 0x9E3779B97F4A7C15ull;   // xorshift64 for sampled n
  auto next = [&state]() {
    state ^= state << 13;
    state ^= state >> 7;
    state ^= state << 17;
    return static_cast<uint32_t>(state >> 32);
  };
  long cases = 0;
  for (uint32_t d : ds) {
    const fp8bs::InvariantDiv inv = fp8bs::invariant_div(d);
    const uint32_t top = 0xFFFFFFFFu;
    for (uint32_t n : {0u, 1u, d - 1, d, d + 1, top, top - 1, top - d, top / d * d,
                       top / d * d - 1, 0x80000000u, 0x7FFFFFFFu}) {
      if (!check_one(n, d, inv)) return 1;
      ++cases;
    }
    // around multiples k * d spread over the whole range
    const uint64_t kmax = top / d;
    for (int i = 0; i < 64; ++i) {
      const uint64_t k = kmax <= 64 ? static_cast<uint64_t>(i) % (kmax + 1)
                                    : (static_cast<uint64_t>(next()) % kmax);
      const uint64_t base = k * d;
      for (int64_t off = -1; off <= 1; ++off) {
        const int64_t v = static_cast<int64_t>(base) + off;
        if (v < 0 || v > static_cast<int64_t>(top)) continue;
        if (!check_one(static_cast<uint32_t>(v), d, inv)) return 1;
        ++cases;
      }
    }
    for (int i = 0; i < 64; ++i) {
      if (!check_one(next(), d, inv)) return 1;
      ++cases;
    }
  }
  {
    const uint32_t d = 7;
    const fp8bs::InvariantDiv inv = fp8bs::invariant_div(d);
    uint32_t n = 0;
    do {
      if (fp8bs::div_invariant(n, inv) != n / d) {
        check_one(n, d, inv);
        return 1;
      }
    } while (++n != 0);
    cases += 1l << 32;
  }
  std::printf("ok %ld quotients\n", cases);
  return 0;
}
