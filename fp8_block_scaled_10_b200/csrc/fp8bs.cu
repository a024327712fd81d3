// C ABI of libfp8bs.so (declared in include/fp8bs.h): argument checks, launch
// configuration, TMA descriptors and the per-device error word.  The kernels
// live in quant.cuh (act_quant, weight_dequant, weight_quant, split-K
// reduction), gemm.cuh (FP8 GEMM with FP32 promotion), gemm_bs.cuh (FP8 GEMM
// on the block-scaled MMA) and transpose.cuh (FP8 transpose, transposing
// quantizer); plan.h plans the dense GEMM launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8bs.h"
#include "gemm.cuh"
#include "gemm_bs.cuh"
#include "plan.h"
#include "quant.cuh"
#include "sm100.cuh"
#include "transpose.cuh"

namespace fp8bs {
namespace {

thread_local char t_last_error[512] = "";

fp8bs_status fail(fp8bs_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

fp8bs_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FP8BS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Opts the GEMM kernel into its dynamic shared memory and checks that the
// registers it is launched with cover its warpgroup register split (a split
// larger than the launch total would make setmaxnreg.inc wait forever).
template <int BN, bool G, int AR = 128, bool BROW = false, bool CHECK = false, bool FUSED = false>
fp8bs_status setup_gemm_kernel() {
  using C = gemm::Cfg<BN, AR>;
  auto kernel = gemm::fp8_gemm_kernel<BN, G, AR, BROW, CHECK, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::smem_bytes(G));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  if (C::kSplitRegs) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
    const long launch_total = static_cast<long>(fa.numRegs) * C::kThreads;
    const long split_total = 128L * C::kCtrlRegs + 32L * C::kEpiWarps * C::kEpiRegs;
    if (fa.numRegs > 168 || split_total > launch_total)
      return fail(FP8BS_ERR_UNSUPPORTED,
                  "GEMM BN=%d register split %ld exceeds launch total %ld (%d regs/thread)", BN,
                  split_total, launch_total, fa.numRegs);
  }
  return FP8BS_OK;
}

template <int BN, bool G, bool BROW = false>
fp8bs_status setup_gemm_bs_kernel() {
  const cudaError_t e =
      cudaFuncSetAttribute(gemm::fp8_gemm_bs_kernel<BN, G, BROW>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gemm::BsCfg<BN>::smem_bytes(G));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return FP8BS_OK;
}

// One-time per-device setup: SM count, shared-memory opt-in of the GEMM
// kernels, and the driver's tensor-map encoder.
fp8bs_status device_setup(int* dev_out, DeviceInfo** info_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8BS_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(FP8BS_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                  dev, major, minor);
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    fp8bs_status r;
    if ((r = setup_gemm_kernel<128, false>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<192, false>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 64>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 64>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 16>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 16>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<128, false>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<256, false>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<128, true>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<256, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 128, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 16, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 16, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 64, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 64, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 128, true>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<128, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_bs_kernel<256, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<128, false, 128, false, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<192, false, 128, false, false, true>()) != FP8BS_OK ||
        (r = setup_gemm_kernel<256, false, 128, false, false, true>()) != FP8BS_OK)
      return r;
    for (auto k : {act_quant_transposed_tma_kernel<false>, act_quant_transposed_tma_kernel<true>}) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               2 * kAqtStageBytes + 1024);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (act_quant_transposed)");
    }
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *dev_out = dev;
  *info_out = &d;
  return FP8BS_OK;
}

// 2-D tensor map over a row-major uint8 matrix [rows, cols] read in boxes of
// [box_rows, 128] with the 128-byte swizzle; out-of-range rows read as zero.
fp8bs_status make_tmap(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                       int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t elem[2] = {1u, 1u};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                              strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FP8BS_OK;
}

// Every GEMM configuration fits the 227 KB of shared memory a CTA can opt into.
constexpr int kMaxSmemOptin = 227 * 1024;
static_assert(gemm::Cfg<256>::smem_bytes(true) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<192>::smem_bytes(false) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<256, 64>::smem_bytes(false) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<128, 64>::smem_bytes(false) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<256, 16>::smem_bytes(false) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<128, 16>::smem_bytes(false) <= kMaxSmemOptin, "smem");
static_assert(gemm::Cfg<128>::smem_bytes(true) <= kMaxSmemOptin, "smem");
static_assert(gemm::BsCfg<256>::smem_bytes(true) <= kMaxSmemOptin, "smem");
static_assert(gemm::BsCfg<128>::smem_bytes(true) <= kMaxSmemOptin, "smem");

// Output map of the GEMM epilogue's TMA stores.  One split: bf16 y [rows,
// cols] in boxes of 32 rows x 32 columns (needs cols % 8 == 0, a 16-byte row
// pitch).  Several: the FP32 workspace [splits][rows][cols] in boxes of 32
// rows x 16 columns of one split (needs cols % 4 == 0), so rows past M are
// clipped inside each split; an FP32 y with one split is mapped the same way
// as a workspace of one split (ws = y).  Both in the 64-byte swizzle the
// epilogue stages them in.  Otherwise *map is zeroed and the kernel stores
// directly (y_tma = 0).
fp8bs_status make_tmap_out(CUtensorMap* map, const void* y, const void* ws, int64_t rows,
                           int64_t cols, int splits, int* y_tma, bool out_f32 = false) {
  memset(map, 0, sizeof(*map));
  *y_tma = 0;
  CUresult r;
  if (splits == 1 && out_f32) ws = y;
  if (splits == 1 && !out_f32) {
    if (cols % 8 != 0) return FP8BS_OK;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2u};
    const cuuint32_t box[2] = {32u, 32u};
    const cuuint32_t elem[2] = {1u, 1u};
    r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(y), dims, strides, box,
                 elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled (y) failed (%d)", (int)r);
    *y_tma = 1;
    return FP8BS_OK;
  }
  if (cols % 4 != 0) return FP8BS_OK;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(splits)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4u,
                                 static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols) * 4u};
  const cuuint32_t box[3] = {16u, 32u, 1u};
  const cuuint32_t elem[3] = {1u, 1u, 1u};
  r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ws), dims, strides, box,
               elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled (ws) failed (%d)", (int)r);
  *y_tma = 2;
  return FP8BS_OK;
}

// Launches a library kernel with programmatic stream serialization: it may
// start while the previous kernel of the stream finishes (every kernel here
// waits for that kernel before touching global memory, and lets the next one
// start early), which overlaps launch latency and prologues across the
// act_quant -> GEMM -> split-K reduction chain.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(n);
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// log2 of a supported quantization block size (32, 64, 128 or 256), else -1.
int block_log2(int64_t block) {
  switch (block) {
    case 32: return 5;
    case 64: return 6;
    case 128: return 7;
    case 256: return 8;
  }
  return -1;
}

template <typename T, bool UE>
cudaError_t launch_act_quant(int64_t block, int grid, cudaStream_t st, const T* x, uint8_t* q,
                             float* s, int64_t nblocks) {
  switch (block) {
    case 32: return launch(act_quant_kernel<T, UE, 32>, grid, kActThreads, 0, st, x, q, s, nblocks);
    case 64: return launch(act_quant_kernel<T, UE, 64>, grid, kActThreads, 0, st, x, q, s, nblocks);
    case 256: return launch(act_quant_kernel<T, UE, 256>, grid, kActThreads, 0, st, x, q, s, nblocks);
    default: return launch(act_quant_kernel<T, UE, 128>, grid, kActThreads, 0, st, x, q, s, nblocks);
  }
}

int grid_for(int64_t work_items, int64_t per_cta, int max_ctas) {
  const int64_t need = (work_items + per_cta - 1) / per_cta;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(need, max_ctas)));
}


// The x map of fused launches; unused (zero) in every other GEMM launch.
const CUtensorMap kNoMap{};

template <int BN, bool G, int AR = 128, bool BROW = false, bool CHECK = false, bool FUSED = false>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tw, const CUtensorMap& ty,
                        const gemm::Params& p, int grid, cudaStream_t st,
                        const CUtensorMap& tx = kNoMap) {
  using C = gemm::Cfg<BN, AR>;
  return launch(gemm::fp8_gemm_kernel<BN, G, AR, BROW, CHECK, FUSED>, grid, C::kThreads,
                C::smem_bytes(G), st, ta, tw, ty, tx, p);
}

// Rows of A one pipeline stage loads: all 128 rows of a tile, or for
// decode-sized M (dense calls only) 16 or 64.
int a_rows_for(int64_t M) { return M <= 16 ? 16 : (M <= 64 ? 64 : 128); }

template <bool G>
cudaError_t launch_gemm_any(int bn, int a_rows, const CUtensorMap& ta, const CUtensorMap& tw,
                            const CUtensorMap& ty, const gemm::Params& p, int grid,
                            cudaStream_t st) {
  // Grouped launches use 128-row A stages and 128- or 256-wide tiles only, so
  // the other variants are not instantiated for them.
  if constexpr (G) {
    (void)a_rows;
    return bn == 256 ? launch_gemm<256, G>(ta, tw, ty, p, grid, st)
                     : launch_gemm<128, G>(ta, tw, ty, p, grid, st);
  } else {
    if (a_rows == 16)
      return bn == 256 ? launch_gemm<256, G, 16>(ta, tw, ty, p, grid, st)
                       : launch_gemm<128, G, 16>(ta, tw, ty, p, grid, st);
    if (a_rows == 64)
      return bn == 256 ? launch_gemm<256, G, 64>(ta, tw, ty, p, grid, st)
                       : launch_gemm<128, G, 64>(ta, tw, ty, p, grid, st);
    return bn == 256 ? launch_gemm<256, G>(ta, tw, ty, p, grid, st)
           : bn == 192 ? launch_gemm<192, G>(ta, tw, ty, p, grid, st)
                       : launch_gemm<128, G>(ta, tw, ty, p, grid, st);
  }
}

// Work units and tile indices are 32-bit in the kernels: the number of
// 128 x 128 output tiles (the most any plan has before a K split, which the
// planner caps at 16) must stay below 2^26.
bool gemm_too_large(int64_t M, int64_t N) {
  return ((M + 127) / 128) * ((N + 127) / 128) >= (int64_t(1) << 26);
}

fp8bs_status check_gemm_operands(const uint8_t* a, const float* a_s, const uint8_t* w,
                                 const float* w_s, const void* y, int64_t N, int64_t K) {
  if (!a || !a_s || !w || !w_s || !y) return fail(FP8BS_ERR_INVALID_ARG, "null operand pointer");
  if (K <= 0 || K % 128 != 0) return fail(FP8BS_ERR_INVALID_ARG, "K=%lld must be a positive multiple of 128", (long long)K);
  if (N <= 0 || N > (1 << 30)) return fail(FP8BS_ERR_INVALID_ARG, "N=%lld out of range", (long long)N);
  if (!aligned16(a) || !aligned16(w) || !aligned16(y))
    return fail(FP8BS_ERR_INVALID_ARG, "a, w and y must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(a_s) & 3u) || (reinterpret_cast<uintptr_t>(w_s) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "scale pointers must be 4-byte aligned");
  return FP8BS_OK;
}

fp8bs_status run_gemm(const uint8_t* a, const float* a_s, const uint8_t* w, const float* w_s,
                      int64_t M, int64_t N, int64_t K, void* y, void* ws, size_t ws_bytes,
                      cudaStream_t st, bool out_f32 = false,
                      bool w_rowwise = false, bool check_pow2 = false, int stall_step = 0) {
  fp8bs_status r = check_gemm_operands(a, a_s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M < 0 || M > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M out of range");
  if (gemm_too_large(M, N)) return fail(FP8BS_ERR_INVALID_ARG, "M x N too large (tile count)");
  if (M == 0) return FP8BS_OK;
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  const Plan pl = plan_gemm(M, N, K, info->sms, w_rowwise ? GemmKind::kRowScaled : GemmKind::kPromotion);
  // Row scales on W: both scale tables are staged K-block-major after the
  // split-K area of the workspace.
  const size_t split_bytes = plan_workspace(pl, M, N);
  const size_t stage_off = (split_bytes + 255) & ~static_cast<size_t>(255);
  const size_t need = w_rowwise ? stage_off + rowwise_stage_bytes(M, N, K) : split_bytes;
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(FP8BS_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required", need);

  CUtensorMap ta, tw, ty;
  gemm::Params p{};
  // Decode-sized M loads only the rows it has; 192-wide tiles are planned for
  // M > 128 only.
  const int a_rows = (pl.bn == 192 || w_rowwise) ? 128 : a_rows_for(M);
  if ((r = make_tmap(&ta, a, M, K, a_rows)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, N, K, pl.bn)) != FP8BS_OK) return r;
  if ((r = make_tmap_out(&ty, y, ws, M, N, pl.splits, &p.y_tma, out_f32)) != FP8BS_OK) return r;
  p.sa = a_s;
  p.sw = w_s;
  if (w_rowwise) {
    float* sa_t = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + stage_off);
    float* sw_t = sa_t + M * (K / 128);
    const int64_t tiles = ((M + 31) / 32 + (N + 31) / 32) * ((K / 128 + 31) / 32);
    const cudaError_t se = launch(scale_tables_kmajor_kernel, grid_for(tiles, 1, info->sms * 8),
                                  dim3(32, 8), 0, st, a_s, sa_t, M, w_s, sw_t, N,
                                  static_cast<int>(K / 128));
    if (se != cudaSuccess) return cuda_fail(se, "scale staging launch");
    p.sa = sa_t;
    p.sw = sw_t;
  }
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.ws = static_cast<float*>(out_f32 && pl.splits == 1 ? y : ws);
  p.out_f32 = out_f32 ? 1 : 0;
  p.m_offsets = nullptr;
  p.stall_step = stall_step;
  set_schedule(p, pl, M, N, K);
  p.tail_ws = pl.tail_splits > 0 ? static_cast<float*>(ws) : nullptr;
  cudaError_t e;
  if (w_rowwise)
    e = pl.bn == 256 ? launch_gemm<256, false, 128, true>(ta, tw, ty, p, pl.grid, st)
                     : launch_gemm<128, false, 128, true>(ta, tw, ty, p, pl.grid, st);
  else if (check_pow2 && (a_rows == 16 || a_rows == 64))
    e = a_rows == 16
            ? (pl.bn == 256 ? launch_gemm<256, false, 16, false, true>(ta, tw, ty, p, pl.grid, st)
                            : launch_gemm<128, false, 16, false, true>(ta, tw, ty, p, pl.grid, st))
            : (pl.bn == 256 ? launch_gemm<256, false, 64, false, true>(ta, tw, ty, p, pl.grid, st)
                            : launch_gemm<128, false, 64, false, true>(ta, tw, ty, p, pl.grid, st));
  else if (check_pow2)
    return fail(FP8BS_ERR_UNSUPPORTED, "scale check without decode tiles (M=%lld)", (long long)M);
  else
    e = launch_gemm_any<false>(pl.bn, a_rows, ta, tw, ty, p, pl.grid, st);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm launch");
  if (pl.tail_splits > 0) {
    const int64_t items = static_cast<int64_t>(pl.tail_tiles) * 128 * (pl.bn / 4);
    e = out_f32
            ? launch(gemm::tail_reduce_kernel<float>, grid_for(items, 256, info->sms * 8), 256, 0,
                     st, static_cast<const float*>(ws), static_cast<float*>(y), M,
                     static_cast<int>(N), pl.m_tiles, pl.n_tiles, pl.n_group, pl.full_units,
                     pl.tail_tiles, pl.tail_splits, pl.bn)
            : launch(gemm::tail_reduce_kernel<__nv_bfloat16>, grid_for(items, 256, info->sms * 8),
                     256, 0, st, static_cast<const float*>(ws),
                     reinterpret_cast<__nv_bfloat16*>(y), M, static_cast<int>(N), pl.m_tiles,
                     pl.n_tiles, pl.n_group, pl.full_units, pl.tail_tiles, pl.tail_splits, pl.bn);
    if (e != cudaSuccess) return cuda_fail(e, "split-tail reduce launch");
  }
  if (pl.splits > 1) {
    const int64_t MN = M * N;
    e = out_f32 ? launch(splitk_reduce_kernel<float>, grid_for(MN, 256 * 4, info->sms * 8), 256,
                         0, st, static_cast<const float*>(ws), static_cast<float*>(y), MN,
                         pl.splits)
                : launch(splitk_reduce_kernel<__nv_bfloat16>, grid_for(MN, 256 * 4, info->sms * 8),
                         256, 0, st, static_cast<const float*>(ws),
                         reinterpret_cast<__nv_bfloat16*>(y), MN, pl.splits);
    if (e != cudaSuccess) return cuda_fail(e, "split-K reduce launch");
  }
  return FP8BS_OK;
}

template <int BN, bool G, bool BROW = false>
cudaError_t launch_gemm_bs(const CUtensorMap& ta, const CUtensorMap& tw, const CUtensorMap& ty,
                           const gemm::Params& p, int grid, cudaStream_t st) {
  using C = gemm::BsCfg<BN>;
  return launch(gemm::fp8_gemm_bs_kernel<BN, G, BROW>, grid, C::kThreads, C::smem_bytes(G), st,
                ta, tw, ty, p);
}

// Block-scaled (ue8m0) GEMM: the same plan as the promotion kernel.
fp8bs_status run_gemm_bs(const uint8_t* a, const float* a_s, const uint8_t* w, const float* w_s,
                         int64_t M, int64_t N, int64_t K, void* y, void* ws, size_t ws_bytes,
                         cudaStream_t st, bool out_f32 = false,
                         bool w_rowwise = false) {
  fp8bs_status r = check_gemm_operands(a, a_s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M < 0 || M > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M out of range");
  if (gemm_too_large(M, N)) return fail(FP8BS_ERR_INVALID_ARG, "M x N too large (tile count)");
  if (M == 0) return FP8BS_OK;
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  const Plan pl = plan_gemm(M, N, K, info->sms, GemmKind::kBlockScaled);
  // Row scales on W: both scale tables are staged K-block-major after the
  // split-K area of the workspace.
  const size_t split_bytes = plan_workspace(pl, M, N);
  const size_t stage_off = (split_bytes + 255) & ~static_cast<size_t>(255);
  const size_t need = w_rowwise ? stage_off + rowwise_stage_bytes(M, N, K) : split_bytes;
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(FP8BS_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required", need);
  CUtensorMap ta, tw, ty;
  gemm::Params p{};
  if ((r = make_tmap(&ta, a, M, K, 128)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, N, K, pl.bn)) != FP8BS_OK) return r;
  if ((r = make_tmap_out(&ty, y, ws, M, N, pl.splits, &p.y_tma, out_f32)) != FP8BS_OK) return r;
  p.sa = a_s;
  p.sw = w_s;
  if (w_rowwise) {
    float* sa_t = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + stage_off);
    float* sw_t = sa_t + M * (K / 128);
    const int64_t tiles = ((M + 31) / 32 + (N + 31) / 32) * ((K / 128 + 31) / 32);
    const cudaError_t se = launch(scale_tables_kmajor_kernel, grid_for(tiles, 1, info->sms * 8),
                                  dim3(32, 8), 0, st, a_s, sa_t, M, w_s, sw_t, N,
                                  static_cast<int>(K / 128));
    if (se != cudaSuccess) return cuda_fail(se, "scale staging launch");
    p.sa = sa_t;
    p.sw = sw_t;
  }
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.ws = static_cast<float*>(out_f32 && pl.splits == 1 ? y : ws);
  p.out_f32 = out_f32 ? 1 : 0;
  p.m_offsets = nullptr;
  set_schedule(p, pl, M, N, K);
  p.tail_ws = pl.tail_splits > 0 ? static_cast<float*>(ws) : nullptr;
  cudaError_t e = w_rowwise
                      ? (pl.bn == 256 ? launch_gemm_bs<256, false, true>(ta, tw, ty, p, pl.grid, st)
                                      : launch_gemm_bs<128, false, true>(ta, tw, ty, p, pl.grid, st))
                      : (pl.bn == 256 ? launch_gemm_bs<256, false>(ta, tw, ty, p, pl.grid, st)
                                      : launch_gemm_bs<128, false>(ta, tw, ty, p, pl.grid, st));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_ue8m0 launch");
  if (pl.tail_splits > 0) {
    const int64_t items = static_cast<int64_t>(pl.tail_tiles) * 128 * (pl.bn / 4);
    e = out_f32
            ? launch(gemm::tail_reduce_kernel<float>, grid_for(items, 256, info->sms * 8), 256, 0,
                     st, static_cast<const float*>(ws), static_cast<float*>(y), M,
                     static_cast<int>(N), pl.m_tiles, pl.n_tiles, pl.n_group, pl.full_units,
                     pl.tail_tiles, pl.tail_splits, pl.bn)
            : launch(gemm::tail_reduce_kernel<__nv_bfloat16>, grid_for(items, 256, info->sms * 8),
                     256, 0, st, static_cast<const float*>(ws),
                     reinterpret_cast<__nv_bfloat16*>(y), M, static_cast<int>(N), pl.m_tiles,
                     pl.n_tiles, pl.n_group, pl.full_units, pl.tail_tiles, pl.tail_splits, pl.bn);
    if (e != cudaSuccess) return cuda_fail(e, "split-tail reduce launch");
  }
  if (pl.splits > 1) {
    const int64_t MN = M * N;
    e = out_f32 ? launch(splitk_reduce_kernel<float>, grid_for(MN, 256 * 4, info->sms * 8), 256,
                         0, st, static_cast<const float*>(ws), static_cast<float*>(y), MN,
                         pl.splits)
                : launch(splitk_reduce_kernel<__nv_bfloat16>, grid_for(MN, 256 * 4, info->sms * 8),
                         256, 0, st, static_cast<const float*>(ws),
                         reinterpret_cast<__nv_bfloat16*>(y), MN, pl.splits);
    if (e != cudaSuccess) return cuda_fail(e, "split-K reduce launch");
  }
  return FP8BS_OK;
}

// Power-of-two (ue8m0) scales.  Decode-sized M (up to 64 rows) runs the
// promotion kernel, whose narrow A stages keep the weight stream at HBM speed
// (the block-scaled kernel loads 128-row A tiles and measured 20-35 % slower
// there); it checks the scales' form as it loads them, as the block-scaled
// kernel does.  Larger M runs the block-scaled MMA.
fp8bs_status run_gemm_pow2(const uint8_t* a, const float* a_s, const uint8_t* w,
                           const float* w_s, int64_t M, int64_t N, int64_t K, void* y, void* ws,
                           size_t ws_bytes, cudaStream_t st, bool out_f32 = false) {
  if (M <= 64)
    return run_gemm(a, a_s, w, w_s, M, N, K, y, ws, ws_bytes, st, out_f32, false, true);
  return run_gemm_bs(a, a_s, w, w_s, M, N, K, y, ws, ws_bytes, st, out_f32);
}

// CTAs of `kernel` that fit on one SM at once (at least 1): persistent
// kernels that loop over tiles are launched with that many per SM.
template <typename K>
int resident_ctas(K kernel, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 1;
  }
  return n > 0 ? n : 1;
}

// y = decode(q) * scale over an M x N code matrix, the scale of (row, col)
// being s[(row >> row_shift) * s_row_stride + (col >> lb)].
cudaError_t launch_dequant(const uint8_t* q, const float* s, int64_t M, int64_t N,
                           int64_t s_row_stride, int row_shift, int lb, void* y, bool bf,
                           int sms, cudaStream_t st) {
  if (N % 16 == 0 && M * (N / 16) < (int64_t(1) << 32) - kDeqThreads * kDeqUnroll * 8 * 1024) {
    const uint32_t cpr = static_cast<uint32_t>(N / 16);
    const uint32_t total = static_cast<uint32_t>(M * (N / 16));
    const int grid = grid_for(total, kDeqThreads * kDeqUnroll, sms * 16);
    const InvariantDiv row_div = invariant_div(cpr);
    return bf ? launch(weight_dequant_kernel<true>, grid, kDeqThreads, 0, st, q, s, y, total, cpr,
                       row_div, s_row_stride, row_shift, lb)
              : launch(weight_dequant_kernel<false>, grid, kDeqThreads, 0, st, q, s, y, total,
                       cpr, row_div, s_row_stride, row_shift, lb);
  }
  const int grid = grid_for(M * N, kDeqThreads, sms * 8);
  return bf ? launch(weight_dequant_any_kernel<true>, grid, kDeqThreads, 0, st, q, s, y, M, N,
                     s_row_stride, row_shift, lb)
            : launch(weight_dequant_any_kernel<false>, grid, kDeqThreads, 0, st, q, s, y, M, N,
                     s_row_stride, row_shift, lb);
}

fp8bs_status run_act_quant(const void* x, fp8bs_dtype x_dtype, int64_t rows, int64_t cols,
                           int64_t block, fp8bs_scale_fmt fmt, uint8_t* q, float* s,
                           cudaStream_t st) {
  if (block_log2(block) < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (rows < 0 || cols <= 0 || cols % block != 0)
    return fail(FP8BS_ERR_INVALID_ARG, "cols=%lld must be a positive multiple of block", (long long)cols);
  if (x_dtype != FP8BS_DTYPE_BF16 && x_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "x_dtype");
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "scale_fmt");
  if (rows == 0) return FP8BS_OK;
  if (!x || !q || !s) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "x and q must be 16-byte aligned, s 4-byte aligned");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const int64_t nblocks = rows * (cols / block);
  // Each thread holds 32 elements: kActThreads * 32 / block blocks per CTA per
  // step; up to 8 CTAs per SM.
  const int grid = grid_for(nblocks, (kActThreads * kActElems / block) * kActUnroll, info->sms * 8);
  const bool ue = fmt == FP8BS_SCALE_FMT_UE8M0;
  cudaError_t e;
  if (x_dtype == FP8BS_DTYPE_BF16) {
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    e = ue ? launch_act_quant<__nv_bfloat16, true>(block, grid, st, xb, q, s, nblocks)
           : launch_act_quant<__nv_bfloat16, false>(block, grid, st, xb, q, s, nblocks);
  } else {
    const auto* xf = static_cast<const float*>(x);
    e = ue ? launch_act_quant<float, true>(block, grid, st, xf, q, s, nblocks)
           : launch_act_quant<float, false>(block, grid, st, xf, q, s, nblocks);
  }
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  return FP8BS_OK;
}

// The fused linear launch (linear.cuh): lp.gemm_ctas CTAs run the GEMM's
// tiles (one wave, no K split), the remaining CTAs quantize x into q and s and
// count each chunk into the flags, which are zeroed first.
fp8bs_status run_linear_fused(const uint16_t* x, int64_t M, int64_t K, bool ue8m0,
                              const uint8_t* w, const float* w_s, int64_t N, uint16_t* y,
                              uint8_t* q, float* s, int* flags, size_t flag_bytes,
                              const LinearPlan& lp, int sms, cudaStream_t st) {
  fp8bs_status r;
  const Plan& pl = lp.gemm;
  CUtensorMap ta, tw, ty, tx;
  gemm::Params p{};
  if ((r = make_tmap(&ta, q, M, K, 128)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, N, K, pl.bn)) != FP8BS_OK) return r;
  if ((r = make_tmap_out(&ty, y, nullptr, M, N, 1, &p.y_tma)) != FP8BS_OK) return r;
  {
    // x [M, K] bf16 in boxes of 128 rows x 64 columns, 128-byte swizzle.
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2u};
    const cuuint32_t box[2] = {64u, 128u};
    const cuuint32_t elem[2] = {1u, 1u};
    const CUresult cr = g_encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x),
                                 dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled (x) failed (%d)", (int)cr);
  }
  p.sa = s;
  p.sw = w_s;
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.ws = nullptr;
  p.m_offsets = nullptr;
  set_schedule(p, pl, M, N, K);
  p.gemm_ctas = lp.gemm_ctas;
  p.fq_flags = flags;
  p.fq_q = q;
  p.fq_s = s;
  p.fq_ue8m0 = ue8m0 ? 1 : 0;
  cudaError_t e = cudaMemsetAsync(flags, 0, flag_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "fused linear flag reset");
  const int grid = lp.gemm_ctas + lp.quant_ctas;
  if (grid > sms) return fail(FP8BS_ERR_UNSUPPORTED, "fused linear grid %d > %d SMs", grid, sms);
  e = pl.bn == 256 ? launch_gemm<256, false, 128, false, false, true>(ta, tw, ty, p, grid, st, tx)
      : pl.bn == 192 ? launch_gemm<192, false, 128, false, false, true>(ta, tw, ty, p, grid, st, tx)
                     : launch_gemm<128, false, 128, false, false, true>(ta, tw, ty, p, grid, st, tx);
  if (e != cudaSuccess) return cuda_fail(e, "fused linear launch");
  return FP8BS_OK;
}

}  // namespace
}  // namespace fp8bs

using namespace fp8bs;

extern "C" {

int fp8bs_version(void) { return 100; }

const char* fp8bs_status_string(fp8bs_status status) {
  switch (status) {
    case FP8BS_OK: return "FP8BS_OK";
    case FP8BS_ERR_INVALID_ARG: return "FP8BS_ERR_INVALID_ARG";
    case FP8BS_ERR_UNSUPPORTED: return "FP8BS_ERR_UNSUPPORTED";
    case FP8BS_ERR_WORKSPACE: return "FP8BS_ERR_WORKSPACE";
    case FP8BS_ERR_CUDA: return "FP8BS_ERR_CUDA";
    case FP8BS_ERR_TIMEOUT: return "FP8BS_ERR_TIMEOUT";
    case FP8BS_ERR_SCALE: return "FP8BS_ERR_SCALE";
  }
  return "FP8BS_UNKNOWN_STATUS";
}

const char* fp8bs_last_error_message(void) { return t_last_error; }

fp8bs_status fp8bs_get_device_error(void* stream, int* code) {
  if (!code) return fail(FP8BS_ERR_INVALID_ARG, "code is null");
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  }
  *code = v;
  return FP8BS_OK;
}

fp8bs_status fp8bs_act_quant(const void* x, fp8bs_dtype x_dtype, int64_t rows, int64_t cols,
                             int64_t block, fp8bs_scale_fmt fmt, uint8_t* q, float* s,
                             void* stream) {
  return run_act_quant(x, x_dtype, rows, cols, block, fmt, q, s, as_stream(stream));
}

fp8bs_status fp8bs_weight_dequant(const uint8_t* q, const float* s, int64_t M, int64_t N,
                                  int64_t block, void* y, fp8bs_dtype y_dtype, void* stream) {
  const int lb = block_log2(block);
  if (lb < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (M < 0 || N < 0) return fail(FP8BS_ERR_INVALID_ARG, "negative size");
  if (y_dtype != FP8BS_DTYPE_BF16 && y_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "y_dtype");
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!q || !s || !y) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(y) || (reinterpret_cast<uintptr_t>(s) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "q and y must be 16-byte aligned, s 4-byte aligned");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const int64_t nbn = (N + block - 1) / block;
  const cudaError_t e = launch_dequant(q, s, M, N, nbn, lb, lb, y, y_dtype == FP8BS_DTYPE_BF16,
                                       info->sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight_dequant launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_act_dequant(const uint8_t* q, const float* s, int64_t s_row_stride,
                               int64_t rows, int64_t cols, int64_t block, void* y,
                               fp8bs_dtype y_dtype, void* stream) {
  const int lb = block_log2(block);
  if (lb < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (rows < 0 || cols <= 0 || cols % block != 0)
    return fail(FP8BS_ERR_INVALID_ARG, "cols=%lld must be a positive multiple of block", (long long)cols);
  if (s_row_stride != 0 && s_row_stride < cols / block)
    return fail(FP8BS_ERR_INVALID_ARG, "s_row_stride=%lld must be 0 or at least cols / block",
                (long long)s_row_stride);
  if (y_dtype != FP8BS_DTYPE_BF16 && y_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "y_dtype");
  if (rows == 0) return FP8BS_OK;
  if (!q || !s || !y) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(y) || (reinterpret_cast<uintptr_t>(s) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "q and y must be 16-byte aligned, s 4-byte aligned");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const cudaError_t e = launch_dequant(q, s, rows, cols, s_row_stride, 0, lb, y,
                                       y_dtype == FP8BS_DTYPE_BF16, info->sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "act_dequant launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_fp8_transpose(const uint8_t* q, const float* s, int64_t R, int64_t C,
                                 int64_t block, uint8_t* qt, float* st, void* stream) {
  if (block_log2(block) < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (R < 0 || C < 0) return fail(FP8BS_ERR_INVALID_ARG, "negative size");
  if (R == 0 || C == 0) return FP8BS_OK;
  if (!q || !s || !qt || !st) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(qt) || (reinterpret_cast<uintptr_t>(s) & 3u) ||
      (reinterpret_cast<uintptr_t>(st) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "q and qt must be 16-byte aligned, s and st 4-byte aligned");
  if (q == qt) return fail(FP8BS_ERR_INVALID_ARG, "the transpose is not in place");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const int64_t sr = (R + block - 1) / block, sc = (C + block - 1) / block;
  cudaStream_t stm = as_stream(stream);
  cudaError_t e;
  if (R % 16 == 0 && C % 16 == 0) {
    const int64_t tiles = ((R + 127) / 128) * ((C + 127) / 128);
    const int per_sm = resident_ctas(fp8_transpose_kernel, kTrThreads, 0);
    e = launch(fp8_transpose_kernel, grid_for(tiles, 1, info->sms * per_sm), kTrThreads, 0, stm,
               q, s, qt, st, R, C, sr, sc);
  } else {
    e = launch(fp8_transpose_any_kernel, grid_for(R * C, 256, info->sms * 8), 256, 0, stm, q, s,
               qt, st, R, C, sr, sc);
  }
  if (e != cudaSuccess) return cuda_fail(e, "fp8_transpose launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_act_quant_transposed(const void* x, fp8bs_dtype x_dtype, int64_t rows,
                                        int64_t cols, int64_t block, fp8bs_scale_fmt fmt,
                                        uint8_t* qt, float* st, void* stream) {
  if (block != 128)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (the transposed quantizer implements 128)",
                (long long)block);
  if (rows < 0 || rows % 128 != 0)
    return fail(FP8BS_ERR_INVALID_ARG, "rows=%lld must be a multiple of 128", (long long)rows);
  if (cols <= 0) return fail(FP8BS_ERR_INVALID_ARG, "cols=%lld", (long long)cols);
  if (cols % 8 != 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "cols=%lld (multiples of 8 are implemented)", (long long)cols);
  if (x_dtype != FP8BS_DTYPE_BF16 && x_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "x_dtype");
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "scale_fmt");
  if (rows == 0) return FP8BS_OK;
  if (!x || !qt || !st) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(qt) || (reinterpret_cast<uintptr_t>(st) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "x and qt must be 16-byte aligned, st 4-byte aligned");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const int64_t tiles = (rows / 128) * ((cols + 127) / 128);
  cudaStream_t stm = as_stream(stream);
  const bool ue = fmt == FP8BS_SCALE_FMT_UE8M0;
  cudaError_t e;
  if (x_dtype == FP8BS_DTYPE_BF16) {
    // TMA-fed kernel: 128 x 128 bf16 boxes of x (columns past cols read as 0)
    CUtensorMap tx;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2u};
    const cuuint32_t box[2] = {128u, 128u};
    const cuuint32_t elem[2] = {1u, 1u};
    const CUresult cr = g_encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x),
                                 dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled (x) failed (%d)", (int)cr);
    const size_t smem = 2 * kAqtStageBytes + 1024;
    const int per_sm = resident_ctas(act_quant_transposed_tma_kernel<false>, kAqtThreads, smem);
    const int grid = grid_for(tiles, 1, info->sms * per_sm);
    e = ue ? launch(act_quant_transposed_tma_kernel<true>, grid, kAqtThreads, smem, stm, tx, qt,
                    st, rows, cols)
           : launch(act_quant_transposed_tma_kernel<false>, grid, kAqtThreads, smem, stm, tx, qt,
                    st, rows, cols);
  } else {
    const int per_sm = resident_ctas(act_quant_transposed_kernel<float, false>, kAqtThreads, 0);
    const int grid = grid_for(tiles, 1, info->sms * per_sm);
    const auto* xf = static_cast<const float*>(x);
    e = ue ? launch(act_quant_transposed_kernel<float, true>, grid, kAqtThreads, 0, stm, xf, qt,
                    st, rows, cols)
           : launch(act_quant_transposed_kernel<float, false>, grid, kAqtThreads, 0, stm, xf, qt,
                    st, rows, cols);
  }
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_transposed launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_act_quant_static(const void* x, fp8bs_dtype x_dtype, int64_t rows,
                                    int64_t cols, int64_t block, const float* s,
                                    int64_t s_row_stride, uint8_t* q, float* s_out,
                                    void* stream) {
  const int lb = block_log2(block);
  if (lb < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (rows < 0 || cols <= 0 || cols % block != 0)
    return fail(FP8BS_ERR_INVALID_ARG, "cols=%lld must be a positive multiple of block", (long long)cols);
  if (s_row_stride != 0 && s_row_stride < cols / block)
    return fail(FP8BS_ERR_INVALID_ARG, "s_row_stride=%lld must be 0 or at least cols / block",
                (long long)s_row_stride);
  if (x_dtype != FP8BS_DTYPE_BF16 && x_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "x_dtype");
  if (rows == 0) return FP8BS_OK;
  if (!x || !s || !q) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s) & 3u) ||
      (reinterpret_cast<uintptr_t>(s_out) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "x and q must be 16-byte aligned, s and s_out 4-byte aligned");
  const int64_t chunks = rows * (cols / kStaticElems);
  if (chunks >= (int64_t(1) << 32) - int64_t(kStaticThreads) * kStaticUnroll * 8 * 1024)
    return fail(FP8BS_ERR_INVALID_ARG, "rows * cols too large");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const uint32_t cpr = static_cast<uint32_t>(cols / kStaticElems);
  const uint32_t total = static_cast<uint32_t>(chunks);
  const int grid = grid_for(total, kStaticThreads * kStaticUnroll, info->sms * 8);
  const InvariantDiv row_div = invariant_div(cpr);
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  if (x_dtype == FP8BS_DTYPE_BF16)
    e = launch(act_quant_static_kernel<__nv_bfloat16>, grid, kStaticThreads, 0, st,
               static_cast<const __nv_bfloat16*>(x), s, q, s_out, total, cpr, row_div,
               s_row_stride, cols / block, lb);
  else
    e = launch(act_quant_static_kernel<float>, grid, kStaticThreads, 0, st,
               static_cast<const float*>(x), s, q, s_out, total, cpr, row_div, s_row_stride,
               cols / block, lb);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_static launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_weight_quant(const void* w, fp8bs_dtype w_dtype, int64_t M, int64_t N,
                                int64_t block, fp8bs_scale_fmt fmt, uint8_t* q, float* s,
                                void* stream) {
  const int lb = block_log2(block);
  if (lb < 0)
    return fail(FP8BS_ERR_UNSUPPORTED, "block=%lld (32, 64, 128 and 256 are implemented)", (long long)block);
  if (M < 0 || N < 0) return fail(FP8BS_ERR_INVALID_ARG, "negative size");
  if (w_dtype != FP8BS_DTYPE_BF16 && w_dtype != FP8BS_DTYPE_F32)
    return fail(FP8BS_ERR_INVALID_ARG, "w_dtype");
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "scale_fmt");
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!w || !q || !s) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  const int64_t rb = (M + block - 1) / block, cb = (N + block - 1) / block;
  if (rb > 65535 || cb > 0x7FFFFFFF) return fail(FP8BS_ERR_INVALID_ARG, "matrix too large");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  const dim3 grid(static_cast<unsigned>(cb), static_cast<unsigned>(rb));
  const bool ue = fmt == FP8BS_SCALE_FMT_UE8M0;
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  if (block == 128) {
    // One pass with the tile in registers; rows of 16 (bf16) or 8 (fp32)
    // bytes per 4 elements must be aligned for the vector loads.
    const size_t esz = w_dtype == FP8BS_DTYPE_F32 ? 4 : 2;
    const bool vec_ok = (N % 4) == 0 && (reinterpret_cast<uintptr_t>(w) % (4 * esz)) == 0 &&
                        (reinterpret_cast<uintptr_t>(q) % 4) == 0;
    e = w_dtype == FP8BS_DTYPE_F32
            ? launch(weight_quant128_kernel<float>, grid, 256, 0, st, static_cast<const float*>(w),
                     q, s, M, N, cb, ue, vec_ok)
            : launch(weight_quant128_kernel<__nv_bfloat16>, grid, 256, 0, st,
                     static_cast<const __nv_bfloat16*>(w), q, s, M, N, cb, ue, vec_ok);
    if (e != cudaSuccess) return cuda_fail(e, "weight_quant launch");
    return FP8BS_OK;
  }
  if (w_dtype == FP8BS_DTYPE_F32)
    e = launch(weight_quant_kernel<float>, grid, 256, 0, st, static_cast<const float*>(w), q, s,
               M, N, cb, ue, lb);
  else
    e = launch(weight_quant_kernel<__nv_bfloat16>, grid, 256, 0, st,
               static_cast<const __nv_bfloat16*>(w), q, s, M, N, cb, ue, lb);
  if (e != cudaSuccess) return cuda_fail(e, "weight_quant launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_selftest_quotient(const float* x, const float* s, float* q, int64_t n,
                                     void* stream) {
  if (n < 0) return fail(FP8BS_ERR_INVALID_ARG, "negative size");
  if (n == 0) return FP8BS_OK;
  if (!x || !s || !q) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  quotient_selftest_kernel<<<grid_for(n, 256, info->sms * 8), 256, 0, as_stream(stream)>>>(x, s, q, n);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quotient self-test launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_selftest_block_scale(const float* amax, float* s, int64_t n, int scale_fmt,
                                        void* stream) {
  if (n < 0) return fail(FP8BS_ERR_INVALID_ARG, "negative size");
  if (scale_fmt != FP8BS_SCALE_FMT_NONE && scale_fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "unknown scale_fmt");
  if (n == 0) return FP8BS_OK;
  if (!amax || !s) return fail(FP8BS_ERR_INVALID_ARG, "null pointer");
  int dev;
  DeviceInfo* info;
  fp8bs_status r = device_setup(&dev, &info);
  if (r != FP8BS_OK) return r;
  scale_selftest_kernel<<<grid_for(n, 256, info->sms * 8), 256, 0, as_stream(stream)>>>(
      amax, s, n, scale_fmt == FP8BS_SCALE_FMT_UE8M0);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "block-scale self-test launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_selftest_gemm_stall(const uint8_t* a, const float* a_s, const uint8_t* w,
                                       const float* w_s, int64_t M, int64_t N, int64_t K,
                                       uint16_t* y, void* workspace, size_t workspace_bytes,
                                       int stall_step, void* stream) {
  if (stall_step < 1) return fail(FP8BS_ERR_INVALID_ARG, "stall_step must be >= 1");
  return run_gemm(a, a_s, w, w_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream),
                  false, false, false, stall_step);
}

size_t fp8bs_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0) return 0;
  int dev;
  DeviceInfo* info;
  if (device_setup(&dev, &info) != FP8BS_OK) return 0;
  // One size serves both GEMM entry points (their plans may differ).
  return std::max({plan_workspace(plan_gemm(M, N, K, info->sms), M, N),
                   plan_workspace(plan_gemm(M, N, K, info->sms, GemmKind::kBlockScaled), M, N),
                   plan_workspace(plan_gemm(M, N, K, info->sms, GemmKind::kRowScaled), M, N)});
}

size_t fp8bs_gemm_rowwise_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0) return 0;
  int dev;
  DeviceInfo* info;
  if (device_setup(&dev, &info) != FP8BS_OK) return 0;
  const size_t split = std::max(
      plan_workspace(plan_gemm(M, N, K, info->sms, GemmKind::kRowScaled), M, N),
      plan_workspace(plan_gemm(M, N, K, info->sms, GemmKind::kBlockScaled), M, N));
  return ((split + 255) & ~static_cast<size_t>(255)) + rowwise_stage_bytes(M, N, K);
}

const char* fp8bs_gemm_plan_string(int64_t M, int64_t N, int64_t K) {
  thread_local char buf[256];
  int dev;
  DeviceInfo* info;
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0 || device_setup(&dev, &info) != FP8BS_OK) {
    snprintf(buf, sizeof(buf), "none");
    return buf;
  }
  const Plan pl = plan_gemm(M, N, K, info->sms);
  snprintf(buf, sizeof(buf),
           "bn=%d m_tiles=%d n_tiles=%d splits=%d kb_per_split=%d units=%d grid=%d sms=%d "
           "tail_tiles=%d tail_splits=%d n_group=%d",
           pl.bn, pl.m_tiles, pl.n_tiles, pl.splits, pl.kb_per_split, pl.units, pl.grid,
           info->sms, pl.tail_tiles, pl.tail_splits, pl.n_group);
  return buf;
}

fp8bs_status fp8bs_fp8_gemm(const uint8_t* a, const float* a_s, const uint8_t* w,
                            const float* w_s, int64_t M, int64_t N, int64_t K, uint16_t* y,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return run_gemm(a, a_s, w, w_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fp8_gemm without a caller workspace: the split-K partials live in this
// file-scope device array, which every GPU that loads the library holds
// until the process exits.  Host code must not pass the array's name to a
// kernel (on the host it is only a stand-in symbol); the device address is
// looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
namespace {
static __device__ __align__(256) float g_static_scratch[FP8BS_STATIC_SCRATCH_BYTES / sizeof(float)];

std::mutex g_scratch_mu;
void* g_scratch_ptr[fp8bs::kMaxDevices] = {};

fp8bs_status static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fp8bs::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= fp8bs::kMaxDevices)
    return fp8bs::fail(FP8BS_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fp8bs::cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                              "cudaGetSymbolAddress(static scratch)");
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return FP8BS_OK;
}
}  // namespace

extern "C" {

fp8bs_status fp8bs_fp8_gemm_static_scratch(const uint8_t* a, const float* a_s, const uint8_t* w,
                                           const float* w_s, int64_t M, int64_t N, int64_t K,
                                           uint16_t* y, void* stream) {
  const size_t need = fp8bs_gemm_workspace_size(M, N, K);
  if (need > FP8BS_STATIC_SCRATCH_BYTES)
    return fp8bs::fail(FP8BS_ERR_WORKSPACE,
                       "M=%lld N=%lld K=%lld needs %zu bytes of split-K scratch; the static "
                       "scratch holds %zu bytes (use fp8bs_fp8_gemm with a workspace)",
                       (long long)M, (long long)N, (long long)K, need,
                       (size_t)FP8BS_STATIC_SCRATCH_BYTES);
  // An empty problem is validated and returns before the scratch is looked up.
  if (M == 0) return fp8bs_fp8_gemm(a, a_s, w, w_s, M, N, K, y, nullptr, 0, stream);
  void* scratch = nullptr;
  const fp8bs_status r = static_scratch_address(&scratch);
  if (r != FP8BS_OK) return r;
  return fp8bs_fp8_gemm(a, a_s, w, w_s, M, N, K, y, scratch, FP8BS_STATIC_SCRATCH_BYTES, stream);
}

fp8bs_status fp8bs_fp8_gemm_ue8m0(const uint8_t* a, const float* a_s, const uint8_t* w,
                                  const float* w_s, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return run_gemm_pow2(a, a_s, w, w_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream));
}

fp8bs_status fp8bs_fp8_gemm_f32(const uint8_t* a, const float* a_s, const uint8_t* w,
                                const float* w_s, int64_t M, int64_t N, int64_t K,
                                fp8bs_scale_fmt fmt, float* y, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fp8bs::fail(FP8BS_ERR_INVALID_ARG, "scale format %d", (int)fmt);
  if (fmt == FP8BS_SCALE_FMT_UE8M0)
    return run_gemm_pow2(a, a_s, w, w_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream),
                         true);
  return run_gemm(a, a_s, w, w_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream), true);
}

fp8bs_status fp8bs_fp8_gemm_rowwise(const uint8_t* a, const float* a_s, const uint8_t* b,
                                    const float* b_s, int64_t M, int64_t N, int64_t K,
                                    fp8bs_scale_fmt fmt, void* y, fp8bs_dtype y_dtype,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fp8bs::fail(FP8BS_ERR_INVALID_ARG, "scale format %d", (int)fmt);
  if (y_dtype != FP8BS_DTYPE_BF16 && y_dtype != FP8BS_DTYPE_F32)
    return fp8bs::fail(FP8BS_ERR_INVALID_ARG, "y_dtype");
  const bool f32 = y_dtype == FP8BS_DTYPE_F32;
  if (fmt == FP8BS_SCALE_FMT_UE8M0)
    return run_gemm_bs(a, a_s, b, b_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream),
                       f32, true);
  return run_gemm(a, a_s, b, b_s, M, N, K, y, workspace, workspace_bytes, as_stream(stream), f32,
                  true);
}

fp8bs_status fp8bs_fp8_linear_ue8m0(const uint16_t* x, int64_t M, int64_t K, const uint8_t* w,
                                    const float* w_s, int64_t N, uint16_t* y, uint8_t* q,
                                    float* s, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  fp8bs_status r = check_gemm_operands(q, s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M == 0) return FP8BS_OK;
  cudaStream_t st = as_stream(stream);
  if ((r = run_act_quant(x, FP8BS_DTYPE_BF16, M, K, 128, FP8BS_SCALE_FMT_UE8M0, q, s, st)) !=
      FP8BS_OK)
    return r;
  return run_gemm_pow2(q, s, w, w_s, M, N, K, y, workspace, workspace_bytes, st);
}

fp8bs_status fp8bs_fp8_gemm_grouped_ue8m0(int64_t G, const int64_t* m_offsets, int64_t M_total,
                                          const uint8_t* a, const float* a_s, const uint8_t* w,
                                          const float* w_s, int64_t N, int64_t K, uint16_t* y,
                                          void* stream) {
  if (G < 1 || G > gemm::kMaxGroups)
    return fail(FP8BS_ERR_INVALID_ARG, "G=%lld out of [1, %d]", (long long)G, gemm::kMaxGroups);
  if (!m_offsets || (reinterpret_cast<uintptr_t>(m_offsets) & 7u))
    return fail(FP8BS_ERR_INVALID_ARG, "m_offsets must be an 8-byte aligned device pointer");
  fp8bs_status r = check_gemm_operands(a, a_s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M_total < 0 || M_total >= (int64_t(1) << 31))
    return fail(FP8BS_ERR_INVALID_ARG, "M_total out of range");
  if (M_total == 0) return FP8BS_OK;
  if (G * N > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "G*N too large");
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  const int bn = N >= 256 ? 256 : 128;
  CUtensorMap ta, tw, ty;
  gemm::Params p{};
  if ((r = make_tmap(&ta, a, M_total, K, 128)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, G * N, K, bn)) != FP8BS_OK) return r;
  if ((r = make_tmap_out(&ty, y, nullptr, M_total, N, 1, &p.y_tma)) != FP8BS_OK) return r;
  p.sa = a_s;
  p.sw = w_s;
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.ws = nullptr;
  p.m_offsets = m_offsets;
  p.M = M_total;
  p.N = static_cast<int>(N);
  p.kbn = static_cast<int>(K / 128);
  p.nbn = static_cast<int>((N + 127) / 128);
  p.m_tiles = 0;
  p.n_tiles = static_cast<int>((N + bn - 1) / bn);
  p.n_group = 1;
  p.splits = 1;
  p.kb_per_split = p.kbn;
  p.num_units = 0;
  p.groups = static_cast<int>(G);
  const int64_t max_units = ((M_total + 127) / 128 + G) * p.n_tiles;
  if (max_units >= (int64_t(1) << 26))
    return fail(FP8BS_ERR_INVALID_ARG, "M_total x N too large (tile count)");
  const int grid = static_cast<int>(std::min<int64_t>(max_units, info->sms));
  cudaError_t e = bn == 256 ? launch_gemm_bs<256, true>(ta, tw, ty, p, grid, as_stream(stream))
                            : launch_gemm_bs<128, true>(ta, tw, ty, p, grid, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_grouped_ue8m0 launch");
  return FP8BS_OK;
}

fp8bs_status fp8bs_fp8_linear(const uint16_t* x, int64_t M, int64_t K, fp8bs_scale_fmt fmt,
                              const uint8_t* w, const float* w_s, int64_t N, uint16_t* y,
                              uint8_t* q, float* s, void* workspace, size_t workspace_bytes,
                              void* stream) {
  fp8bs_status r = check_gemm_operands(q, s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M < 0 || M > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M out of range");
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "scale_fmt");
  if (M == 0) return FP8BS_OK;
  cudaStream_t st = as_stream(stream);
  if (x != nullptr && aligned16(x) && !gemm_too_large(M, N)) {
    int dev;
    DeviceInfo* info;
    if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
    const LinearPlan lp = plan_linear(M, N, K, info->sms);
    const size_t flag_bytes = linear_flag_bytes(M, K);
    if (lp.fused && workspace != nullptr && aligned16(workspace) && workspace_bytes >= flag_bytes)
      return run_linear_fused(x, M, K, fmt == FP8BS_SCALE_FMT_UE8M0, w, w_s, N, y, q, s,
                              static_cast<int*>(workspace), flag_bytes, lp, info->sms, st);
  }
  if ((r = run_act_quant(x, FP8BS_DTYPE_BF16, M, K, 128, fmt, q, s, st)) != FP8BS_OK) return r;
  return run_gemm(q, s, w, w_s, M, N, K, y, workspace, workspace_bytes, st);
}

fp8bs_status fp8bs_fp8_linear_fused(const uint16_t* x, int64_t M, int64_t K,
                                    fp8bs_scale_fmt fmt, const uint8_t* w, const float* w_s,
                                    int64_t N, uint16_t* y, uint8_t* q, float* s,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  fp8bs_status r = check_gemm_operands(q, s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (x == nullptr || !aligned16(x)) return fail(FP8BS_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (M < 0 || M > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M out of range");
  if (fmt != FP8BS_SCALE_FMT_NONE && fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "scale_fmt");
  if (M == 0) return FP8BS_OK;
  if (gemm_too_large(M, N)) return fail(FP8BS_ERR_INVALID_ARG, "M x N too large (tile count)");
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  const LinearPlan lp = plan_linear_fused(M, N, K, info->sms);
  if (!lp.fused)
    return fail(FP8BS_ERR_UNSUPPORTED,
                "no fused launch for M=%lld N=%lld: M must exceed 128 and the GEMM's tiles must "
                "leave %d SMs free", (long long)M, (long long)N, kMinQuantCtas);
  const size_t flag_bytes = linear_flag_bytes(M, K);
  if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < flag_bytes)
    return fail(FP8BS_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required", flag_bytes);
  return run_linear_fused(x, M, K, fmt == FP8BS_SCALE_FMT_UE8M0, w, w_s, N, y, q, s,
                          static_cast<int*>(workspace), flag_bytes, lp, info->sms,
                          as_stream(stream));
}

size_t fp8bs_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0) return 0;
  return std::max(fp8bs_gemm_workspace_size(M, N, K), linear_flag_bytes(M, K));
}

const char* fp8bs_linear_plan_string(int64_t M, int64_t N, int64_t K) {
  thread_local char buf[256];
  int dev;
  DeviceInfo* info;
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0 || device_setup(&dev, &info) != FP8BS_OK) {
    snprintf(buf, sizeof(buf), "none");
    return buf;
  }
  const LinearPlan lp = plan_linear(M, N, K, info->sms);
  const LinearPlan f = plan_linear_fused(M, N, K, info->sms);
  char alt[96] = "fused: none";
  if (f.fused)
    snprintf(alt, sizeof(alt), "fused: bn=%d gemm_ctas=%d quant_ctas=%d est_us=%.1f", f.gemm.bn,
             f.gemm_ctas, f.quant_ctas, f.est_us);
  snprintf(buf, sizeof(buf), "%s bn=%d est_us=%.1f | %s", lp.fused ? "fused" : "act_quant+gemm",
           lp.gemm.bn, lp.est_us, alt);
  return buf;
}

fp8bs_status fp8bs_fp8_gemm_grouped(int64_t G, const int64_t* m_offsets, int64_t M_total,
                                    const uint8_t* a, const float* a_s, const uint8_t* w,
                                    const float* w_s, int64_t N, int64_t K, uint16_t* y,
                                    void* stream) {
  if (G < 1 || G > gemm::kMaxGroups) return fail(FP8BS_ERR_INVALID_ARG, "G=%lld out of [1, %d]", (long long)G, gemm::kMaxGroups);
  if (!m_offsets || (reinterpret_cast<uintptr_t>(m_offsets) & 7u))
    return fail(FP8BS_ERR_INVALID_ARG, "m_offsets must be an 8-byte aligned device pointer");
  fp8bs_status r = check_gemm_operands(a, a_s, w, w_s, y, N, K);
  if (r != FP8BS_OK) return r;
  if (M_total < 0 || M_total >= (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M_total out of range");
  if (M_total == 0) return FP8BS_OK;
  if (G * N > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "G*N too large");
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  // The tile width with the least estimated time per 128-row tile of a group
  // (192-wide tiles and the group table do not fit shared memory together).
  int bn = 128;
  for (int cand : {256}) {
    if (N < cand) continue;
    const auto cost = [&](int b) { return ((N + b - 1) / b) * kb_time_us(GemmKind::kPromotion, b); };
    if (cost(cand) < cost(bn) - 1e-9) bn = cand;
  }
  CUtensorMap ta, tw, ty;
  gemm::Params p{};
  if ((r = make_tmap(&ta, a, M_total, K, 128)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, G * N, K, bn)) != FP8BS_OK) return r;
  if ((r = make_tmap_out(&ty, y, nullptr, M_total, N, 1, &p.y_tma)) != FP8BS_OK) return r;
  p.sa = a_s;
  p.sw = w_s;
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.ws = nullptr;
  p.m_offsets = m_offsets;
  p.M = M_total;
  p.N = static_cast<int>(N);
  p.kbn = static_cast<int>(K / 128);
  p.nbn = static_cast<int>((N + 127) / 128);
  p.m_tiles = 0;
  p.n_tiles = static_cast<int>((N + bn - 1) / bn);
  p.n_group = 1;
  p.splits = 1;
  p.kb_per_split = p.kbn;
  p.num_units = 0;
  p.groups = static_cast<int>(G);
  // Units are only known on the device; an upper bound sizes the grid.
  const int64_t max_units = ((M_total + 127) / 128 + G) * p.n_tiles;
  if (max_units >= (int64_t(1) << 26))
    return fail(FP8BS_ERR_INVALID_ARG, "M_total x N too large (tile count)");
  const int grid = static_cast<int>(std::min<int64_t>(max_units, info->sms));
  cudaError_t e = launch_gemm_any<true>(bn, 128, ta, tw, ty, p, grid, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_grouped launch");
  return FP8BS_OK;
}

}  // extern "C"

extern "C" {

fp8bs_status fp8bs_fp8_gemm_quant(const uint8_t* a, const float* a_s, const uint8_t* w,
                                  const float* w_s, int64_t M, int64_t N, int64_t K,
                                  fp8bs_scale_fmt out_fmt, uint8_t* q_out, float* s_out,
                                  uint16_t* y, void* stream) {
  fp8bs_status r = check_gemm_operands(a, a_s, w, w_s, reinterpret_cast<uint16_t*>(q_out), N, K);
  if (r != FP8BS_OK) return r;
  if (N % 128 != 0)
    return fail(FP8BS_ERR_INVALID_ARG, "N=%lld must be a multiple of 128 (1x128 output blocks)",
                (long long)N);
  if (out_fmt != FP8BS_SCALE_FMT_NONE && out_fmt != FP8BS_SCALE_FMT_UE8M0)
    return fail(FP8BS_ERR_INVALID_ARG, "out_fmt");
  if (s_out == nullptr || (reinterpret_cast<uintptr_t>(s_out) & 3u))
    return fail(FP8BS_ERR_INVALID_ARG, "s_out must be a 4-byte aligned device pointer");
  if (y != nullptr && !aligned16(y)) return fail(FP8BS_ERR_INVALID_ARG, "y must be 16-byte aligned");
  if (M < 0 || M > (int64_t(1) << 31)) return fail(FP8BS_ERR_INVALID_ARG, "M out of range");
  if (gemm_too_large(M, N)) return fail(FP8BS_ERR_INVALID_ARG, "M x N too large (tile count)");
  if (M == 0) return FP8BS_OK;
  int dev;
  DeviceInfo* info;
  if ((r = device_setup(&dev, &info)) != FP8BS_OK) return r;
  // One 128 x 256 tile per unit, no K split: each epilogue thread then owns
  // exactly one 1x128 block of its output row.
  const int bn = 256;
  const int a_rows = a_rows_for(M);
  CUtensorMap ta, tw, tq;
  gemm::Params p{};
  if ((r = make_tmap(&ta, a, M, K, a_rows)) != FP8BS_OK) return r;
  if ((r = make_tmap(&tw, w, N, K, bn)) != FP8BS_OK) return r;
  {
    // q_out [M, N] uint8 in boxes of 32 rows x 64 codes, 64-byte swizzle.
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N)};
    const cuuint32_t box[2] = {64u, 32u};
    const cuuint32_t elem[2] = {1u, 1u};
    const CUresult cr = g_encode(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_out, dims, strides, box,
                                 elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(FP8BS_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)cr);
  }
  const int m_tiles = static_cast<int>((M + 127) / 128);
  const int n_tiles = static_cast<int>((N + bn - 1) / bn);
  const int64_t units = static_cast<int64_t>(m_tiles) * n_tiles;
  if (units > (int64_t(1) << 31) - 1) return fail(FP8BS_ERR_INVALID_ARG, "problem too large");
  p.sa = a_s;
  p.sw = w_s;
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.M = M;
  p.N = static_cast<int>(N);
  p.kbn = static_cast<int>(K / 128);
  p.nbn = static_cast<int>((N + 127) / 128);
  p.m_tiles = m_tiles;
  p.n_tiles = n_tiles;
  p.n_group = choose_n_group(M, K, bn, n_tiles);
  p.splits = 1;
  p.kb_per_split = p.kbn;
  p.num_units = static_cast<int>(units);
  p.groups = 1;
  p.y_tma = 3;
  p.q_out = q_out;
  p.s_out = s_out;
  p.q_ue8m0 = out_fmt == FP8BS_SCALE_FMT_UE8M0 ? 1 : 0;
  const int grid = static_cast<int>(std::min<int64_t>(units, info->sms));
  const cudaError_t e = launch_gemm_any<false>(bn, a_rows, ta, tw, tq, p, grid, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_gemm_quant launch");
  return FP8BS_OK;
}

}  // extern "C"
