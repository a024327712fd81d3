// Compile-time (static_assert) and host check of the GEMM kernels' resource
// budgets, for every configuration the library launches:
//   - dynamic shared memory within the 227 KB a B200 CTA can opt into;
//   - the control block fits its reserved bytes;
//   - TMEM: the partial buffers (or the accumulators and scale-factor ring)
//     fit the 512 columns allocated;
//   - every tile slot starts on a 1024-byte boundary (128-byte swizzle);
//   - the warp register split fits the registers the block launches with;
//   - with 16- or 64-row A stages, the 128-row A operand the MMA reads from
//     the last stage stays inside the CTA's allocation.
// Built and run on the CPU by tests/test_kernel_budgets.py; prints "ok".
#include <cstdio>

#include "gemm.cuh"
#include "gemm_bs.cuh"

namespace {

using namespace fp8bs::gemm;

constexpr int kMaxSmem = 227 * 1024;   // per-CTA opt-in limit on sm_100
constexpr int kLaunchRegCap = 168;     // __launch_bounds__(384, 1): 65536 / 384, rounded down to 8

template <int BN, int ARows, bool G>
constexpr bool promotion_ok() {
  using C = Cfg<BN, ARows>;
  static_assert(C::smem_bytes(G) <= kMaxSmem, "shared memory");
  static_assert(sizeof(Ctrl<C::kStages>) <= C::kCtrlBytes, "control block");
  static_assert(C::kAccBufs <= 4 && C::kAccBufs <= C::kScaleSlots, "TMEM buffers vs barriers");
  static_assert(C::kAccBufs * BN <= C::kTmemCols && C::kTmemCols <= 512, "TMEM columns");
  static_assert(C::kABytes % 1024 == 0 && C::kBBytes % 1024 == 0, "swizzle alignment");
  static_assert(!C::kSplitRegs ||
                    128 * C::kCtrlRegs + 32 * C::kEpiWarps * C::kEpiRegs <= C::kThreads * kLaunchRegCap,
                "register split");
  static_assert(C::kCtrlRegs % 8 == 0 && C::kEpiRegs % 8 == 0 && C::kCtrlRegs >= 24 &&
                    C::kEpiRegs <= 256,
                "setmaxnreg counts");
  // the MMA reads BM rows of A from the last stage's A slot onwards
  static_assert((C::kStages - 1) * C::kABytes + BM * BK <= C::smem_bytes(G) - 1024,
                "A operand over-read stays in the allocation");
  return true;
}

template <int BN, bool G>
constexpr bool block_scaled_ok() {
  using C = BsCfg<BN>;
  static_assert(C::smem_bytes(G) <= kMaxSmem, "shared memory");
  static_assert(sizeof(BsCtrl<C::kStages>) <= C::kCtrlBytes, "control block");
  static_assert(C::kAccBufs <= 2, "accumulator barriers");
  static_assert(C::kSFBase + C::kSFSlots * C::kSFCols <= C::kTmemCols, "TMEM columns");
  static_assert(C::kABytes % 1024 == 0 && C::kBBytes % 1024 == 0 && C::kSFBytes % 128 == 0,
                "slot alignment");
  return true;
}

}  // namespace

int main() {
  // promotion kernel: dense 128/192/256 x 128-row A, decode 16/64-row A, grouped 128/256
  constexpr bool ok =
      promotion_ok<128, 128, false>() && promotion_ok<192, 128, false>() &&
      promotion_ok<256, 128, false>() && promotion_ok<128, 64, false>() &&
      promotion_ok<256, 64, false>() && promotion_ok<128, 16, false>() &&
      promotion_ok<256, 16, false>() && promotion_ok<128, 128, true>() &&
      promotion_ok<256, 128, true>() && block_scaled_ok<128, false>() &&
      block_scaled_ok<256, false>() && block_scaled_ok<128, true>() &&
      block_scaled_ok<256, true>();
  std::printf(ok ? "ok: promotion smem 128/192/256 = %d/%d/%d B, grouped 256 = %d B, "
                   "block-scaled 256 = %d B\n"
                 : "failed\n",
              Cfg<128>::smem_bytes(false), Cfg<192>::smem_bytes(false),
              Cfg<256>::smem_bytes(false), Cfg<256>::smem_bytes(true),
              BsCfg<256>::smem_bytes(false));
  return ok ? 0 : 1;
}
