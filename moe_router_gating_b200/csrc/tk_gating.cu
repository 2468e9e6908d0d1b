// C ABI of the fused MoE top-k gating library (declared in include/tk_gating.h):
// argument validation, launch planning, TMA descriptor encoding and the calls
// into the launch code, which gating_bf16.cu and gating_fp8.cu instantiate
// (two translation units, compiled in parallel).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tk_gating.h"
#include "gating_launch.cuh"

namespace {

__device__ uint32_t g_tk_error_word = 0;
// SM cycles, nanoseconds and launches of the gating kernels (first CTA of each
// launch), summed until tk_gating_clock_counters clears them.
__device__ uint64_t g_tk_clock[3] = {0, 0, 0};

// bounded-wait limit for kernels launched from here (any host thread may set it)
std::atomic<uint64_t> g_timeout_ns{1000000000ull};

constexpr int kMaxDynamicSmem = tkg::kMaxDynamicSmem;
constexpr int kSmemReserve = 1024 + tkg::EPI_BARRIER_RESERVE;  // 1 KB alignment pad + barriers and flags
constexpr int kMaxStages = 8;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using tkg::round_up;

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

using tkg::split_row_stride;

constexpr int kMaxSplit = 16;  // CTAs per cluster in the split-H variant (16 needs non-portable clusters)

// Split-H plan: one 128-token tile per cluster of C CTAs, single-CTA MMAs.
tk_status plan_split_h(int64_t T, int64_t H, int64_t E, int C, tk_gating_plan* plan) {
  const int n_pad = round_up(static_cast<int>(E), 16);
  const int g_pad = n_pad < tkg::E_GROUP ? n_pad : tkg::E_GROUP;  // MMA N of the (largest) expert group
  // one 64-wide K slice per ring stage: the split-H mainloop is bound by the latency of refilling
  // the ring, and finer stages are refilled sooner (measured 1-3% faster than two slices per
  // stage on the 1- to 4096-token workloads)
  const int kps = 1;
  const int b_boxes = (g_pad + tkg::B_BOX_N - 1) / tkg::B_BOX_N;
  const int stage_bytes = tkg::A_STAGE_BYTES + b_boxes * tkg::B_BOX_BYTES;
  int stages = (kMaxDynamicSmem - kSmemReserve) / (kps * stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  const int row_stride = split_row_stride(E);
  // the staged partial rows of a tile (one 256-expert pass at a time) reuse the ring
  if (stages < 2 || tkg::BLOCK_M * row_stride * 4 > stages * kps * stage_bytes) return TK_ERR_UNSUPPORTED;
  const int64_t tiles = (T + tkg::BLOCK_M - 1) / tkg::BLOCK_M;
  plan->variant = TK_VARIANT_SPLIT_H;
  plan->block_m = tkg::BLOCK_M;
  plan->n_pad = n_pad;
  plan->num_tiles = static_cast<int32_t>(tiles);
  plan->k_blocks = static_cast<int32_t>((H + tkg::BLOCK_K - 1) / tkg::BLOCK_K);
  plan->split_h = C;
  plan->stages = stages;
  plan->grid = static_cast<int32_t>(tiles * C);
  plan->cluster = C;
  plan->threads = tkg::SPLIT_THREADS;
  plan->smem_bytes = stages * kps * stage_bytes + kSmemReserve;
  plan->tmem_cols = static_cast<int32_t>(pow2_at_least(round_up(g_pad, 32)));
  plan->slices_per_stage = kps;
  plan->expert_groups = n_pad > tkg::E_GROUP ? 2 : 1;
  return TK_OK;
}

// Clusters of 2^i CTAs (one CTA per SM) that a device runs at once, i = 0..4.
// Measured on B200 (148 SMs): 148, 74, 33, 15, 7 -- GPCs do not divide evenly
// into 4-, 8- and 16-SM groups.  Scaled for other SM counts when planning
// without a device; launches use the device's own figures.
struct ClusterCapacity {
  int n[5];
};

ClusterCapacity b200_like_capacity(int num_sms) {
  ClusterCapacity c;
  c.n[0] = num_sms;
  c.n[1] = num_sms / 2;
  c.n[2] = num_sms * 33 / 148;
  c.n[3] = num_sms * 15 / 148;
  c.n[4] = num_sms * 7 / 148;
  return c;
}

int log2_of(int c) {
  int i = 0;
  while ((1 << i) < c) ++i;
  return i;
}

tk_status plan_impl(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, const ClusterCapacity& cap,
                    tk_gating_plan* plan) {
  if (plan == nullptr || num_sms < 1) return TK_ERR_INVALID_ARG;
  std::memset(plan, 0, sizeof(*plan));
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) {
    plan->variant = TK_VARIANT_NONE;
    return TK_OK;
  }
  const int64_t tiles128 = (T + tkg::BLOCK_M - 1) / tkg::BLOCK_M;
  const int64_t k_blocks = (H + tkg::BLOCK_K - 1) / tkg::BLOCK_K;
  if (tiles128 * 2 <= num_sms) {
    // Few tiles: a cluster of C CTAs splits H for each 128-token tile; C is the
    // largest size whose clusters all run at once (one wave).
    int C = kMaxSplit;
    while (C > 1 && (tiles128 > cap.n[log2_of(C)] || C > k_blocks)) C >>= 1;
    if (C >= 2) return plan_split_h(T, H, E, C, plan);
  }
  const bool pair = E > 64;  // gate halves of >= 64 experts per CTA (128-byte swizzle blocks)
  const int cg = pair ? 2 : 1;
  const int n_pad = pair ? round_up(static_cast<int>(E), 128) : round_up(static_cast<int>(E), 16);
  const int g_pad = n_pad < tkg::E_GROUP ? n_pad : tkg::E_GROUP;  // MMA N of the (largest) expert group
  const int acc_stride = round_up(g_pad, 32);
  const int acc_bufs = 2 * acc_stride <= 512 ? 2 : 1;  // 512 tensor-memory columns
  const int b_boxes = pair ? g_pad / 2 / tkg::B_BOX_N : (g_pad + tkg::B_BOX_N - 1) / tkg::B_BOX_N;
  const int stage_bytes = tkg::KB_PER_STAGE * (tkg::A_STAGE_BYTES + b_boxes * tkg::B_BOX_BYTES);
  // eight epilogue warps: the hand-over of one column half's top-k lists, 128 rows of
  // KMAX (value, id) pairs
  const int kmax = k <= 4 ? 4 : (k <= 8 ? 8 : (k <= 16 ? 16 : 32));
  const int groups = n_pad > tkg::E_GROUP ? 2 : 1;
  const int hand_bytes = tkg::epi_warps(kmax, groups) == 8 ? tkg::BLOCK_M * kmax * 8 : 0;
  int stages = (kMaxDynamicSmem - kSmemReserve - hand_bytes) / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return TK_ERR_UNSUPPORTED;
  const int64_t rows_per_tile = static_cast<int64_t>(tkg::BLOCK_M) * cg;
  int64_t tiles = (T + rows_per_tile - 1) / rows_per_tile;
  const int64_t units_max = num_sms / cg;  // CTAs (or CTA pairs) resident at once
  const int64_t units = tiles < units_max ? tiles : units_max;
  int64_t half_tiles = 0;
  if (pair) {
    // Balanced tail: count work in 128-row units (a full pair tile is 2).  After
    // F full rounds, if the u units left fit one per pair, run them as half tiles
    // (half the MMA time) instead of a partly idle round of full tiles.
    const int64_t h = (T + tkg::BLOCK_M - 1) / tkg::BLOCK_M;
    const int64_t F = h / (2 * units);
    const int64_t u = h - 2 * units * F;
    if (F >= 1 && u > 0 && u <= units) {
      tiles = F * units;
      half_tiles = u;
    }
  }

  plan->variant = pair ? TK_VARIANT_ROW_PAIRS : TK_VARIANT_ROW_TILES;
  plan->block_m = static_cast<int32_t>(rows_per_tile);
  plan->n_pad = n_pad;
  plan->num_tiles = static_cast<int32_t>(tiles);
  plan->k_blocks = static_cast<int32_t>((H + tkg::BLOCK_K - 1) / tkg::BLOCK_K);
  plan->split_h = 1;
  plan->stages = stages;
  plan->grid = static_cast<int32_t>(units * cg);
  plan->num_half_tiles = static_cast<int32_t>(half_tiles);
  plan->cluster = cg;
  plan->threads = tkg::row_tile_threads(kmax, groups);
  plan->smem_bytes = stages * stage_bytes + kSmemReserve + hand_bytes;
  plan->tmem_cols = static_cast<int32_t>(pow2_at_least(acc_bufs * acc_stride));
  plan->slices_per_stage = tkg::KB_PER_STAGE;
  plan->expert_groups = n_pad > tkg::E_GROUP ? 2 : 1;
  return TK_OK;
}

// Few-token plan (bf16, T <= FEW_MAX_TOKENS): ceil(E / 32) blocks of 32 experts,
// each split in H over h_blocks CTAs of h_rows rows (a multiple of 8), about one
// CTA per SM in all.  TK_ERR_UNSUPPORTED when its shared memory does not fit.
tk_status plan_few_tokens(int64_t T, int64_t H, int64_t E, int32_t num_sms, tk_gating_plan* plan,
                          int64_t* workspace_bytes) {
  const int e_blocks = static_cast<int>((E + tkg::FEW_EXPERTS - 1) / tkg::FEW_EXPERTS);
  int64_t h_blocks = std::max<int64_t>(1, num_sms / e_blocks);
  h_blocks = std::min<int64_t>(h_blocks, H / 8);
  const int64_t h_rows = (H + h_blocks - 1) / h_blocks;
  const int h_rows8 = static_cast<int>((h_rows + 7) / 8 * 8);
  h_blocks = (H + h_rows8 - 1) / h_rows8;  // no empty block
  const int e_pad = e_blocks * tkg::FEW_EXPERTS;
  const tkg::FewTokenSmem lay = tkg::few_token_smem(static_cast<int>(T), h_rows8, static_cast<int>(h_blocks), e_pad);
  if (lay.total > kMaxDynamicSmem) return TK_ERR_UNSUPPORTED;
  std::memset(plan, 0, sizeof(*plan));
  plan->variant = TK_VARIANT_FEW_TOKENS;
  plan->block_m = static_cast<int32_t>(T);
  plan->n_pad = e_pad;
  plan->num_tiles = 1;
  plan->k_blocks = static_cast<int32_t>((H + tkg::BLOCK_K - 1) / tkg::BLOCK_K);
  plan->split_h = static_cast<int32_t>(h_blocks);
  plan->grid = static_cast<int32_t>(h_blocks * e_blocks);
  plan->cluster = 1;
  plan->threads = tkg::FEW_THREADS;
  plan->smem_bytes = lay.total;
  plan->expert_groups = 1;
  plan->h_rows = h_rows8;
  *workspace_bytes = tkg::few_token_workspace_bytes(T, static_cast<int>(h_blocks), e_pad);
  return TK_OK;
}

// The plan of the workspace entry points (tk_gating_fused_topk_ws): the plan
// without workspace, except that
//  * bf16 calls of at most FEW_MAX_TOKENS tokens (E <= 256) run the few-token
//    kernel, whose CTAs combine their partial logits through the workspace;
//  * a last round of half tiles on CTA pairs (one expert group, lists of at
//    most 8) becomes ceil(half tiles / 2) 256-token tiles each split in H
//    between two pairs.
// *workspace_bytes is what the plan needs (0 when it is the plain one).
tk_status plan_impl_ws(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, const ClusterCapacity& cap,
                       bool fp8, tk_gating_plan* plan, int64_t* workspace_bytes) {
  if (workspace_bytes == nullptr) return TK_ERR_INVALID_ARG;
  *workspace_bytes = 0;
  const tk_status st = plan_impl(T, H, E, k, num_sms, cap, plan);
  if (st != TK_OK) return st;
  if (!fp8 && T >= 1 && T <= tkg::FEW_MAX_TOKENS && E <= tkg::FEW_MAX_EXPERTS) {
    tk_gating_plan few;
    int64_t bytes = 0;
    if (plan_few_tokens(T, H, E, num_sms, &few, &bytes) == TK_OK) {
      *plan = few;
      *workspace_bytes = bytes;
      return TK_OK;
    }
  }
  // measured (65536 tokens, E = 256, k = 8; split vs plain): H = 7168 -1.7 to
  // -2.0%, H = 4096 -0.7 to +1.6%, H = 3072 +5.5%, H = 2048 +11%, FP8 H = 7168
  // (56 slices) +4.6 to +13%: the split pays only for long tiles, so it needs 96
  // or more K slices, and E <= 256 (the first half's rows fit the idle ring)
  if (plan->variant != TK_VARIANT_ROW_PAIRS || plan->expert_groups != 1 || k > 8 || plan->num_half_tiles == 0 ||
      plan->k_blocks < 96 || E > 256)
    return TK_OK;
  const int split = (plan->num_half_tiles + 1) / 2;  // 256-token tiles; at most half the pairs take one each
  if (2 * split > plan->grid / 2) return TK_OK;
  plan->num_split_tiles = split;
  plan->split_k_block = round_up((plan->k_blocks + 1) / 2, tkg::KB_PER_STAGE);
  plan->num_half_tiles = 0;
  *workspace_bytes = tkg::split_workspace_bytes(split, E);
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

// 2-D uint8 (FP8 E4M3 bits) row-major [rows, cols] map with a (box_cols x
// box_rows) box, 128-byte swizzle: a box row of 128 values is one swizzle row.
bool encode_2d_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estrides[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estrides,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device facts and one-time kernel set-up, filled on the first call made with
// that device current: compute capability, SM count, the device address of the
// error word, every kernel's shared-memory limit (set to the maximum once, so no
// per-call attribute calls), and the largest split-H cluster the device can
// co-schedule.
struct DeviceState {
  bool ready = false;
  tk_status status = TK_OK;
  int num_sms = 0;
  uint32_t* err_word = nullptr;
  uint64_t* clock = nullptr;
  int max_split_cluster = 0;
  ClusterCapacity capacity = {};
};

constexpr int kMaxDevices = 64;
DeviceState g_devices[kMaxDevices];
std::mutex g_devices_mutex;

const DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& d = g_devices[dev];
  std::lock_guard<std::mutex> lock(g_devices_mutex);
  if (d.ready) return &d;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (major != 10 || minor != 0) {
    d.status = TK_ERR_UNSUPPORTED;
    d.ready = true;
    return &d;
  }
  void* err = nullptr;
  void* clk = nullptr;
  if (cudaGetSymbolAddress(&err, g_tk_error_word) != cudaSuccess ||
      cudaGetSymbolAddress(&clk, g_tk_clock) != cudaSuccess || !tkg::set_up_gating_kernels<false>() ||
      !tkg::set_up_gating_kernels<true>()) {
    cudaGetLastError();
    return nullptr;  // not cached: a later call retries
  }
  d.err_word = static_cast<uint32_t*>(err);
  d.clock = static_cast<uint64_t*>(clk);
  d.capacity.n[0] = d.num_sms;
  tkg::measure_split_cluster_capacity(d.capacity.n + 1);
  d.max_split_cluster = 0;
  for (int i = 4; i >= 1; --i)
    if (d.capacity.n[i] > 0) {
      d.max_split_cluster = 1 << i;
      break;
    }
  d.status = TK_OK;
  d.ready = true;
  return &d;
}

// A caller's workspace for the workspace entry points (null: the entry points
// without one).
struct Workspace {
  void* ptr;
  int64_t bytes;
};

// Launch tokens of split last rounds: non-zero, different for every launch.
std::atomic<uint32_t> g_split_token{0};
uint32_t next_split_token() {
  uint32_t t = g_split_token.fetch_add(1, std::memory_order_relaxed) + 1;
  if (t == 0) t = g_split_token.fetch_add(1, std::memory_order_relaxed) + 1;
  return t;
}

// Plan on the current device: without a workspace, or the workspace plan, whose
// bytes the caller's workspace must hold (checked before any launch).
tk_status plan_for_call(int64_t T, int64_t H, int64_t E, int32_t k, const DeviceState* dev, const Workspace* ws,
                        bool fp8, tk_gating_plan* pl) {
  if (ws == nullptr) return plan_impl(T, H, E, k, dev->num_sms, dev->capacity, pl);
  int64_t need = 0;
  const tk_status st = plan_impl_ws(T, H, E, k, dev->num_sms, dev->capacity, fp8, pl, &need);
  if (st != TK_OK) return st;
  if (need > 0 && (ws->ptr == nullptr || ws->bytes < need)) return TK_ERR_INVALID_ARG;
  if (need > 0 && !aligned16(ws->ptr)) return TK_ERR_ALIGNMENT;
  return TK_OK;
}

// route: per-expert counts of the stored ids for the routing that follows
// (tk_gating_fused_topk_route); a null table when nothing is counted.
tk_status fused_topk_device(const void* hidden, const void* gate, int64_t T, int64_t H, int64_t E, int32_t k,
                            float* scores, int32_t* ids, float* logits, cudaStream_t stream,
                            const tkg::RouteCounts& route = tkg::RouteCounts{nullptr, 0u, 0},
                            const Workspace* ws = nullptr) {
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!hidden || !gate || !scores || !ids) return TK_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(gate) || !aligned16(scores) || !aligned16(ids)) return TK_ERR_ALIGNMENT;
  const DeviceState* dev = device_state();
  if (dev == nullptr) return TK_ERR_CUDA;
  if (dev->status != TK_OK) return dev->status;
  tk_gating_plan pl;
  st = plan_for_call(T, H, E, k, dev, ws, false, &pl);
  if (st != TK_OK) return st;

  CUtensorMap mx, mx64, mw;
  std::memset(&mx, 0, sizeof(mx));
  std::memset(&mx64, 0, sizeof(mx64));
  std::memset(&mw, 0, sizeof(mw));
  if (pl.variant != TK_VARIANT_FEW_TOKENS &&  // that kernel reads the inputs with plain loads
      (!encode_2d_bf16(&mx, hidden, static_cast<uint64_t>(T), static_cast<uint64_t>(H), tkg::BLOCK_K,
                       tkg::BLOCK_M) ||
       (pl.num_half_tiles > 0 && !encode_2d_bf16(&mx64, hidden, static_cast<uint64_t>(T),
                                                 static_cast<uint64_t>(H), tkg::BLOCK_K, tkg::BLOCK_M / 2)) ||
       !encode_2d_bf16(&mw, gate, static_cast<uint64_t>(H), static_cast<uint64_t>(E), tkg::B_BOX_N, tkg::BLOCK_K)))
    return TK_ERR_CUDA;
  const tkg::LaunchEnv env{dev->max_split_cluster, dev->err_word, g_timeout_ns.load(std::memory_order_relaxed),
                           dev->clock, route, ws != nullptr ? ws->ptr : nullptr,
                           pl.num_split_tiles > 0 ? next_split_token() : 0u, hidden, gate};
  return tkg::launch_planned<false>(pl, env, mx, mx64, mw, T, H, E, k, scores, ids, nullptr, nullptr, logits, stream);
}

// FP8 sizes: H a multiple of 16 (16-byte rows of 8-bit values); E and k as bf16.
tk_status validate_sizes_fp8(int64_t T, int64_t H, int64_t E, int32_t k) {
  if (T < 0 || H < 1 || E < 1 || k < 1 || k > E) return TK_ERR_INVALID_ARG;
  if (H % 16 != 0) return TK_ERR_UNSUPPORTED;
  return validate_sizes(T, H / 2, E, k);
}

tk_status fused_topk_fp8_device(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k, float* scores,
                                int32_t* ids, float* logits, cudaStream_t stream, const Workspace* ws = nullptr) {
  tk_status st = validate_sizes_fp8(T, H, E, k);
  if (st != TK_OK) return st;
  if (T == 0) return TK_OK;
  if (!hidden_q || !hidden_scale || !gate_q || !gate_scale || !scores || !ids) return TK_ERR_INVALID_ARG;
  if (!aligned16(hidden_q) || !aligned16(gate_q) || !aligned16(scores) || !aligned16(ids) ||
      !aligned16(hidden_scale) || !aligned16(gate_scale))
    return TK_ERR_ALIGNMENT;
  const DeviceState* dev = device_state();
  if (dev == nullptr) return TK_ERR_CUDA;
  if (dev->status != TK_OK) return dev->status;
  // a K slice of 128 FP8 values occupies what 64 bf16 values do: plan on H / 2
  tk_gating_plan pl;
  st = plan_for_call(T, H / 2, E, k, dev, ws, true, &pl);
  if (st != TK_OK) return st;

  CUtensorMap mx, mx64, mw;
  std::memset(&mx64, 0, sizeof(mx64));
  const uint32_t kslice = 2 * tkg::BLOCK_K;  // 128 values: one 128-byte swizzle row
  if (!encode_2d_u8(&mx, hidden_q, static_cast<uint64_t>(T), static_cast<uint64_t>(H), kslice, tkg::BLOCK_M) ||
      (pl.num_half_tiles > 0 &&
       !encode_2d_u8(&mx64, hidden_q, static_cast<uint64_t>(T), static_cast<uint64_t>(H), kslice, tkg::BLOCK_M / 2)) ||
      !encode_2d_u8(&mw, gate_q, static_cast<uint64_t>(E), static_cast<uint64_t>(H), kslice, tkg::B_BOX_N))
    return TK_ERR_CUDA;
  const tkg::LaunchEnv env{dev->max_split_cluster, dev->err_word, g_timeout_ns.load(std::memory_order_relaxed),
                           dev->clock, tkg::RouteCounts{nullptr, 0u, 0}, ws != nullptr ? ws->ptr : nullptr,
                           pl.num_split_tiles > 0 ? next_split_token() : 0u, hidden_q, gate_q};
  return tkg::launch_planned<true>(pl, env, mx, mx64, mw, T, H, E, k, scores, ids, hidden_scale, gate_scale, logits,
                                   stream);
}

}  // namespace

namespace tkg {
// route.cu: the routing half of tk_gating_fused_topk_route
tk_status route_fused_plan(int64_t T, int32_t k, int32_t E, tk_route_plan* pl);
tk_status route_fused_launch(const tk_route_plan& pl, const int32_t* ids, int64_t n, int32_t E, int32_t* workspace,
                             int32_t* offsets, int32_t* sorted_slots, int32_t* slot_pos, cudaStream_t stream);

// The device error word of the current device for the other kernels of this
// library (expert-parallel dispatch and combine); null without an sm_100 device.
uint32_t* device_error_word() {
  const DeviceState* d = device_state();
  return d != nullptr && d->status == TK_OK ? d->err_word : nullptr;
}
}  // namespace tkg

extern "C" {

tk_status tk_gating_fused_topk(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                               int32_t k, float* scores, int32_t* ids, void* stream) {
  return fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, nullptr, static_cast<cudaStream_t>(stream));
}

tk_status tk_gating_fused_topk_ws(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                                  int32_t k, float* scores, int32_t* ids, void* workspace, int64_t workspace_bytes,
                                  void* stream) {
  if (workspace_bytes < 0) return TK_ERR_INVALID_ARG;
  const Workspace ws{workspace, workspace_bytes};
  return fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, nullptr, static_cast<cudaStream_t>(stream),
                           tkg::RouteCounts{nullptr, 0u, 0}, &ws);
}

tk_status tk_gating_fused_topk_ws_logits(const void* hidden, const void* gate_weight, int64_t T, int64_t H,
                                         int64_t E, int32_t k, float* scores, int32_t* ids, float* logits,
                                         void* workspace, int64_t workspace_bytes, void* stream) {
  const tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK || T == 0) return st;
  if (logits == nullptr || workspace_bytes < 0) return TK_ERR_INVALID_ARG;
  if (!aligned16(logits)) return TK_ERR_ALIGNMENT;
  const Workspace ws{workspace, workspace_bytes};
  return fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, logits, static_cast<cudaStream_t>(stream),
                           tkg::RouteCounts{nullptr, 0u, 0}, &ws);
}

tk_status tk_gating_fused_topk_fp8_ws(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                      const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k,
                                      float* scores, int32_t* ids, void* workspace, int64_t workspace_bytes,
                                      void* stream) {
  if (workspace_bytes < 0) return TK_ERR_INVALID_ARG;
  const Workspace ws{workspace, workspace_bytes};
  return fused_topk_fp8_device(hidden_q, hidden_scale, gate_q, gate_scale, T, H, E, k, scores, ids, nullptr,
                               static_cast<cudaStream_t>(stream), &ws);
}

tk_status tk_gating_make_plan_ws(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, tk_gating_plan* plan,
                                 int64_t* workspace_bytes) {
  if (num_sms < 1 || plan == nullptr) return TK_ERR_INVALID_ARG;
  return plan_impl_ws(T, H, E, k, num_sms, b200_like_capacity(num_sms), false, plan, workspace_bytes);
}

tk_status tk_gating_make_plan_fp8_ws(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms,
                                     tk_gating_plan* plan, int64_t* workspace_bytes) {
  if (num_sms < 1 || plan == nullptr) return TK_ERR_INVALID_ARG;
  const tk_status st = validate_sizes_fp8(T, H, E, k);
  if (st != TK_OK) {
    std::memset(plan, 0, sizeof(*plan));
    if (workspace_bytes != nullptr) *workspace_bytes = 0;
    return st;
  }
  return plan_impl_ws(T, H / 2, E, k, num_sms, b200_like_capacity(num_sms), true, plan, workspace_bytes);
}

tk_status tk_gating_workspace_bytes(int64_t T, int64_t H, int64_t E, int32_t k, int32_t fp8,
                                    int64_t* workspace_bytes) {
  if (workspace_bytes == nullptr) return TK_ERR_INVALID_ARG;
  *workspace_bytes = 0;
  const tk_status st = fp8 ? validate_sizes_fp8(T, H, E, k) : validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  const DeviceState* dev = device_state();
  if (dev == nullptr) return TK_ERR_CUDA;
  if (dev->status != TK_OK) return dev->status;
  tk_gating_plan pl;
  return plan_impl_ws(T, fp8 ? H / 2 : H, E, k, dev->num_sms, dev->capacity, fp8 != 0, &pl, workspace_bytes);
}

tk_status tk_gating_fused_topk_logits(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                                      int32_t k, float* scores, int32_t* ids, float* logits, void* stream) {
  const tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK || T == 0) return st;
  if (logits == nullptr) return TK_ERR_INVALID_ARG;
  if (!aligned16(logits)) return TK_ERR_ALIGNMENT;
  return fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, logits, static_cast<cudaStream_t>(stream));
}

tk_status tk_gating_fused_topk_route(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                                     int32_t k, float* scores, int32_t* ids, int32_t* offsets, int32_t* sorted_slots,
                                     int32_t* slot_pos, void* workspace, int64_t workspace_bytes, void* stream) {
  tk_status st = validate_sizes(T, H, E, k);
  if (st != TK_OK) return st;
  if (T > 0 && T > static_cast<int64_t>(INT32_MAX) / k) return TK_ERR_UNSUPPORTED;  // positions are int32
  if (offsets == nullptr) return TK_ERR_INVALID_ARG;
  if (T > 0 && (!hidden || !gate_weight || !scores || !ids || !sorted_slots || !slot_pos)) return TK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0 || (reinterpret_cast<uintptr_t>(sorted_slots) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(slot_pos) & 3u) != 0)
    return TK_ERR_ALIGNMENT;
  if (T > 0 && (!aligned16(hidden) || !aligned16(gate_weight) || !aligned16(scores) || !aligned16(ids)))
    return TK_ERR_ALIGNMENT;
  tk_route_plan rp;  // needs the device's SM count
  st = tkg::route_fused_plan(T, k, static_cast<int32_t>(E), &rp);
  if (st != TK_OK) return st;
  if (rp.fused_workspace_bytes > 0) {
    if (workspace == nullptr || workspace_bytes < rp.fused_workspace_bytes) return TK_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return TK_ERR_ALIGNMENT;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t E4 = static_cast<int32_t>((E + 3) / 4 * 4);
  const tkg::RouteCounts rc{rp.ctas > 1 ? static_cast<int32_t*>(workspace) : nullptr,
                            static_cast<uint32_t>(rp.warp_slots * (rp.threads / 32)), E4};  // a CTA's range: its warps' ranges
  st = fused_topk_device(hidden, gate_weight, T, H, E, k, scores, ids, nullptr, s, rc);
  if (st != TK_OK) return st;
  return tkg::route_fused_launch(rp, ids, T * static_cast<int64_t>(k), static_cast<int32_t>(E),
                                 static_cast<int32_t*>(workspace), offsets, sorted_slots, slot_pos, s);
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
  st = fused_topk_device(hidden_dev, gate_weight, T, H, E, k, scores_dev, ids_dev, nullptr, s);
  if (st != TK_OK) return st;
  if (cudaMemcpyAsync(scores_host, scores_dev, out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(ids_host, ids_dev, out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TK_ERR_CUDA;
  return TK_OK;
}

tk_status tk_gating_fused_topk_fp8(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                   const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k, float* scores,
                                   int32_t* ids, void* stream) {
  return fused_topk_fp8_device(hidden_q, hidden_scale, gate_q, gate_scale, T, H, E, k, scores, ids, nullptr,
                               static_cast<cudaStream_t>(stream));
}

tk_status tk_gating_fused_topk_fp8_logits(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                          const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k,
                                          float* scores, int32_t* ids, float* logits, void* stream) {
  const tk_status st = validate_sizes_fp8(T, H, E, k);
  if (st != TK_OK || T == 0) return st;
  if (logits == nullptr) return TK_ERR_INVALID_ARG;
  if (!aligned16(logits)) return TK_ERR_ALIGNMENT;
  return fused_topk_fp8_device(hidden_q, hidden_scale, gate_q, gate_scale, T, H, E, k, scores, ids, logits,
                               static_cast<cudaStream_t>(stream));
}

tk_status tk_gating_make_plan(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, tk_gating_plan* plan) {
  if (num_sms < 1) return TK_ERR_INVALID_ARG;
  return plan_impl(T, H, E, k, num_sms, b200_like_capacity(num_sms), plan);
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

tk_status tk_gating_clock_counters(uint64_t* sm_cycles, uint64_t* elapsed_ns, uint64_t* launches, int32_t clear) {
  if (sm_cycles == nullptr || elapsed_ns == nullptr || launches == nullptr) return TK_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return TK_ERR_CUDA;
  uint64_t c[3] = {0, 0, 0};
  if (cudaMemcpyFromSymbol(c, g_tk_clock, sizeof(c)) != cudaSuccess) return TK_ERR_CUDA;
  if (clear) {
    const uint64_t zero[3] = {0, 0, 0};
    if (cudaMemcpyToSymbol(g_tk_clock, zero, sizeof(zero)) != cudaSuccess) return TK_ERR_CUDA;
  }
  *sm_cycles = c[0];
  *elapsed_ns = c[1];
  *launches = c[2];
  return TK_OK;
}

tk_status tk_gating_set_wait_timeout_ns(uint64_t timeout_ns) {
  if (timeout_ns < 1000) return TK_ERR_INVALID_ARG;
  g_timeout_ns.store(timeout_ns, std::memory_order_relaxed);
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
