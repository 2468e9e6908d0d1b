// C ABI of the fused MoE top-k gating library (declared in include/tk_gating.h):
// argument validation, launch planning, TMA descriptor encoding and launches.
// The computation itself is in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "tk_gating.h"
#include "gating_row_tiles.cuh"

namespace {

__device__ uint32_t g_tk_error_word = 0;

uint64_t g_timeout_ns = 1000000000ull;  // bounded-wait limit for kernels launched from here

constexpr int kMaxDynamicSmem = 232448;  // 227 KB opt-in per CTA on sm_100
constexpr int kSmemReserve = 1024 + 256;  // 1 KB alignment pad + barriers and flags
constexpr int kMaxStages = 8;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int round_up(int v, int m) { return (v + m - 1) / m * m; }

uint32_t pow2_at_least(uint32_t v) {
  uint32_t c = 32;
  while (c < v) c <<= 1;
  return c;
}

tk_status validate_sizes(int64_t T, int64_t H, int64_t E, int32_t k) {
  if (T < 0 || H < 1 || E < 1 || k < 1 || k > E) return TK_ERR_INVALID_ARG;
  if (H % 8 != 0 || E % 8 != 0) return TK_ERR_UNSUPPORTED;  // 16-byte row pitch for TMA
  if (E < 16 || E > TK_GATING_MAX_EXPERTS || k > TK_GATING_MAX_TOPK) return TK_ERR_UNSUPPORTED;
  if (T > INT32_MAX - tkg::BLOCK_M || H > INT32_MAX - tkg::BLOCK_K) return TK_ERR_UNSUPPORTED;
  return TK_OK;
}

tk_status plan_impl(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, tk_gating_plan* plan) {
  if (plan == nullptr || num_sms < 1) return TK_ERR_INVALID_ARG;
  std::memset(plan, 0, sizeof(*plan));
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) {
    plan->variant = TK_VARIANT_NONE;
    return TK_OK;
  }
  const bool pair = E > 64;  // gate halves of >= 64 experts per CTA (128-byte swizzle blocks)
  const int cg = pair ? 2 : 1;
  const int n_pad = pair ? round_up(static_cast<int>(E), 128) : round_up(static_cast<int>(E), 16);
  const int acc_stride = round_up(n_pad, 32);
  const int b_boxes = pair ? n_pad / 2 / tkg::B_BOX_N : (n_pad + tkg::B_BOX_N - 1) / tkg::B_BOX_N;
  const int stage_bytes = tkg::A_STAGE_BYTES + b_boxes * tkg::B_BOX_BYTES;
  int stages = (kMaxDynamicSmem - kSmemReserve) / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return TK_ERR_UNSUPPORTED;
  const int64_t rows_per_tile = static_cast<int64_t>(tkg::BLOCK_M) * cg;
  const int64_t tiles = (T + rows_per_tile - 1) / rows_per_tile;
  const int64_t units = num_sms / cg;  // CTAs (or CTA pairs) resident at once

  plan->variant = pair ? TK_VARIANT_ROW_PAIRS : TK_VARIANT_ROW_TILES;
  plan->block_m = static_cast<int32_t>(rows_per_tile);
  plan->n_pad = n_pad;
  plan->num_tiles = static_cast<int32_t>(tiles);
  plan->k_blocks = static_cast<int32_t>((H + tkg::BLOCK_K - 1) / tkg::BLOCK_K);
  plan->split_h = 1;
  plan->stages = stages;
  plan->grid = static_cast<int32_t>((tiles < units ? tiles : units) * cg);
  plan->cluster = cg;
  plan->threads = tkg::ROW_TILE_THREADS;
  plan->smem_bytes = stages * stage_bytes + kSmemReserve;
  plan->tmem_cols = static_cast<int32_t>(pow2_at_least(2 * acc_stride));
  return TK_OK;
}

// ---- driver entry point for tensor-map encoding (no link-time libcuda) ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] map with a (box_cols x box_rows) box, 128-byte swizzle.
bool encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estrides[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estrides,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

tk_status check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TK_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TK_ERR_CUDA;
  if (major != 10 || minor != 0) return TK_ERR_UNSUPPORTED;
  return TK_OK;
}

uint32_t* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_tk_error_word) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(p);
}

template <int KMAX, int CG>
tk_status launch_row_tiles(const tk_gating_plan& pl, const CUtensorMap& mx, const CUtensorMap& mw,
                           const tkg::RowTileParams& prm, cudaStream_t stream) {
  auto kernel = tkg::gating_row_tiles_kernel<KMAX, CG>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem_bytes) != cudaSuccess)
    return TK_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = CG > 1 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kernel, mx, mw, prm) != cudaSuccess) return TK_ERR_CUDA;
  return TK_OK;
}

template <int KMAX>
tk_status launch_row_variant(const tk_gating_plan& pl, const CUtensorMap& mx, const CUtensorMap& mw,
                             const tkg::RowTileParams& prm, cudaStream_t stream) {
  if (pl.variant == TK_VARIANT_ROW_PAIRS) return launch_row_tiles<KMAX, 2>(pl, mx, mw, prm, stream);
  return launch_row_tiles<KMAX, 1>(pl, mx, mw, prm, stream);
}

tk_status fused_topk_device(const void* hidden, const void* gate, int64_t T, int64_t H, int64_t E, int32_t k,
                            float* scores, int32_t* ids, cudaStream_t stream) {
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!hidden || !gate || !scores || !ids) return TK_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(gate) || !aligned16(scores) || !aligned16(ids)) return TK_ERR_ALIGNMENT;
  int num_sms = 0;
  st = check_device(&num_sms);
  if (st != TK_OK) return st;
  tk_gating_plan pl;
  st = plan_impl(T, H, E, k, num_sms, &pl);
  if (st != TK_OK) return st;

  CUtensorMap mx, mw;
  if (!encode_2d_bf16(&mx, hidden, static_cast<uint64_t>(T), static_cast<uint64_t>(H), tkg::BLOCK_K,
                      tkg::BLOCK_M) ||
      !encode_2d_bf16(&mw, gate, static_cast<uint64_t>(H), static_cast<uint64_t>(E), tkg::B_BOX_N, tkg::BLOCK_K))
    return TK_ERR_CUDA;
  uint32_t* err = device_error_word();
  if (err == nullptr) return TK_ERR_CUDA;

  tkg::RowTileParams prm;
  prm.T = static_cast<int32_t>(T);
  prm.H = static_cast<int32_t>(H);
  prm.E = static_cast<int32_t>(E);
  prm.k = k;
  prm.n_pad = pl.n_pad;
  prm.acc_stride = round_up(pl.n_pad, 32);
  prm.num_tiles = pl.num_tiles;
  prm.k_blocks = pl.k_blocks;
  prm.stages = pl.stages;
  prm.b_boxes = pl.variant == TK_VARIANT_ROW_PAIRS ? pl.n_pad / 2 / tkg::B_BOX_N
                                                   : (pl.n_pad + tkg::B_BOX_N - 1) / tkg::B_BOX_N;
  prm.tmem_cols = static_cast<uint32_t>(pl.tmem_cols);
  prm.timeout_ns = g_timeout_ns;
  prm.scores = scores;
  prm.ids = ids;
  prm.err_word = err;

  if (k <= 1) return launch_row_variant<1>(pl, mx, mw, prm, stream);
  if (k <= 2) return launch_row_variant<2>(pl, mx, mw, prm, stream);
  if (k <= 4) return launch_row_variant<4>(pl, mx, mw, prm, stream);
  if (k <= 8) return launch_row_variant<8>(pl, mx, mw, prm, stream);
  return launch_row_variant<16>(pl, mx, mw, prm, stream);
}

}  // namespace

extern "C" {

tk_status tk_gating_fused_topk(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                               int32_t k, float* scores, int32_t* ids, void* stream) {
  return fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, static_cast<cudaStream_t>(stream));
}

tk_status tk_gating_fused_topk_host(const void* hidden_host, const void* gate_weight, int64_t T, int64_t H,
                                    int64_t E, int32_t k, float* scores_host, int32_t* ids_host, void* hidden_dev,
                                    float* scores_dev, int32_t* ids_dev, void* stream) {
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!hidden_host || !scores_host || !ids_host) return TK_ERR_INVALID_ARG;
  if (!hidden_dev || !gate_weight || !scores_dev || !ids_dev) return TK_ERR_INVALID_ARG;
  if (!aligned16(hidden_dev) || !aligned16(gate_weight) || !aligned16(scores_dev) || !aligned16(ids_dev))
    return TK_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t in_bytes = static_cast<size_t>(T) * static_cast<size_t>(H) * 2;
  const size_t out_bytes = static_cast<size_t>(T) * static_cast<size_t>(k) * 4;
  if (cudaMemcpyAsync(hidden_dev, hidden_host, in_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return TK_ERR_CUDA;
  st = fused_topk_device(hidden_dev, gate_weight, T, H, E, k, scores_dev, ids_dev, s);
  if (st != TK_OK) return st;
  if (cudaMemcpyAsync(scores_host, scores_dev, out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(ids_host, ids_dev, out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TK_ERR_CUDA;
  return TK_OK;
}

tk_status tk_gating_make_plan(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, tk_gating_plan* plan) {
  return plan_impl(T, H, E, k, num_sms, plan);
}

tk_status tk_gating_device_error(uint32_t* word, int32_t clear) {
  if (word == nullptr) return TK_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return TK_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpyFromSymbol(&w, g_tk_error_word, sizeof(w)) != cudaSuccess) return TK_ERR_CUDA;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_tk_error_word, &zero, sizeof(zero)) != cudaSuccess) return TK_ERR_CUDA;
  }
  *word = w;
  return w ? TK_ERR_DEVICE_TIMEOUT : TK_OK;
}

tk_status tk_gating_set_wait_timeout_ns(uint64_t timeout_ns) {
  if (timeout_ns < 1000) return TK_ERR_INVALID_ARG;
  g_timeout_ns = timeout_ns;
  return TK_OK;
}

const char* tk_gating_status_string(tk_status status) {
  switch (status) {
    case TK_OK: return "TK_OK";
    case TK_ERR_INVALID_ARG: return "TK_ERR_INVALID_ARG: invalid argument";
    case TK_ERR_UNSUPPORTED: return "TK_ERR_UNSUPPORTED: request outside the kernels' supported range or device";
    case TK_ERR_ALIGNMENT: return "TK_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case TK_ERR_CUDA: return "TK_ERR_CUDA: CUDA call failed";
    case TK_ERR_DEVICE_TIMEOUT: return "TK_ERR_DEVICE_TIMEOUT: a kernel wait expired";
  }
  return "unknown tk_status";
}

}  // extern "C"
