// Definitions of the launch interface (gating_launch.cuh): kernel set-up and
// launches, instantiated once per precision by gating_bf16.cu and gating_fp8.cu.
#pragma once

#include "gating_launch.cuh"

namespace tkg {

inline int min_int(int a, int b) { return a < b ? a : b; }

template <typename Kernel>
bool set_smem_limit(Kernel kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynamicSmem) == cudaSuccess;
}

template <int KMAX, bool FP8>
bool set_up_kernels_of() {
  bool ok = set_smem_limit(gating_row_tiles_kernel<KMAX, 1, FP8, 1>) &&
            set_smem_limit(gating_row_tiles_kernel<KMAX, 2, FP8, 1>) &&
            (KMAX > 8 || set_smem_limit(gating_row_tiles_kernel<(KMAX > 8 ? 8 : KMAX), 2, FP8, 1, true>)) &&
            set_smem_limit(gating_row_tiles_kernel<KMAX, 2, FP8, 2>) &&
            set_smem_limit(gating_split_h_kernel<KMAX, 2, FP8>) &&
            set_smem_limit(gating_split_h_kernel<KMAX, 4, FP8>) &&
            set_smem_limit(gating_split_h_kernel<KMAX, 8, FP8>) &&
            set_smem_limit(gating_split_h_kernel<KMAX, 16, FP8>);
  if constexpr (!FP8) ok = ok && set_smem_limit(gating_few_tokens_kernel<KMAX>);
  return ok && cudaFuncSetAttribute(gating_split_h_kernel<KMAX, 16, FP8>,
                                    cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
}

template <bool FP8>
bool set_up_gating_kernels() {
  return set_up_kernels_of<4, FP8>() && set_up_kernels_of<8, FP8>() && set_up_kernels_of<16, FP8>() &&
         set_up_kernels_of<32, FP8>();
}

template <int KMAX, int CG, bool FP8, int EG, bool SPLIT = false>
tk_status launch_row_tiles(const tk_gating_plan& pl, const CUtensorMap& mx, const CUtensorMap& mx64,
                           const CUtensorMap& mw, const RowTileParams& prm, cudaStream_t stream) {
  auto kernel = gating_row_tiles_kernel<KMAX, CG, FP8, EG, SPLIT>;
  // programmatic dependent launch: CTAs may start on SMs the previous kernel has
  // left and set up while it finishes (the producer waits before its loads)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CG;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = CG > 1 ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kernel, mx, mx64, mw, prm) != cudaSuccess) return TK_ERR_CUDA;
  return TK_OK;
}

template <int KMAX, int C, bool FP8>
tk_status launch_split_h_c(const tk_gating_plan& plan, const CUtensorMap& mx, const CUtensorMap& mw,
                           const SplitHParams& prm, cudaStream_t stream) {
  auto kernel = gating_split_h_kernel<KMAX, C, FP8>;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as launch_row_tiles
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.num_tiles * C);
  cfg.blockDim = dim3(plan.threads);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kernel, mx, mw, prm) != cudaSuccess) return TK_ERR_CUDA;
  return TK_OK;
}

template <int KMAX, bool FP8>
tk_status launch_split_h(const tk_gating_plan& plan, int max_cluster, const CUtensorMap& mx, const CUtensorMap& mw,
                         const SplitHParams& prm, cudaStream_t stream) {
  int C = plan.cluster;
  while (C > max_cluster) C >>= 1;  // the largest cluster the device co-schedules
  switch (C) {
    case 16: return launch_split_h_c<KMAX, 16, FP8>(plan, mx, mw, prm, stream);
    case 8: return launch_split_h_c<KMAX, 8, FP8>(plan, mx, mw, prm, stream);
    case 4: return launch_split_h_c<KMAX, 4, FP8>(plan, mx, mw, prm, stream);
    case 2: return launch_split_h_c<KMAX, 2, FP8>(plan, mx, mw, prm, stream);
    default: return TK_ERR_UNSUPPORTED;
  }
}

template <int KMAX>
tk_status launch_few_tokens(const tk_gating_plan& pl, const FewTokenParams& prm, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as launch_row_tiles
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(FEW_THREADS);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gating_few_tokens_kernel<KMAX>, prm) != cudaSuccess) return TK_ERR_CUDA;
  return TK_OK;
}

template <int KMAX, bool FP8>
tk_status launch_row_variant(const tk_gating_plan& pl, const CUtensorMap& mx, const CUtensorMap& mx64,
                             const CUtensorMap& mw, const RowTileParams& prm, cudaStream_t stream) {
  if (pl.variant == TK_VARIANT_ROW_PAIRS) {
    if (pl.expert_groups == 2) return launch_row_tiles<KMAX, 2, FP8, 2>(pl, mx, mx64, mw, prm, stream);
    if constexpr (KMAX <= 8) {
      if (pl.num_split_tiles > 0) return launch_row_tiles<KMAX, 2, FP8, 1, true>(pl, mx, mx64, mw, prm, stream);
    } else {
      if (pl.num_split_tiles > 0) return TK_ERR_UNSUPPORTED;  // the planner splits only lists of <= 8
    }
    return launch_row_tiles<KMAX, 2, FP8, 1>(pl, mx, mx64, mw, prm, stream);
  }
  return launch_row_tiles<KMAX, 1, FP8, 1>(pl, mx, mx64, mw, prm, stream);
}

// Launch the planned kernel on encoded maps.  FP8: hscale / gscale are the
// per-token and per-expert scales (unused for bf16).
template <bool FP8>
tk_status launch_planned(const tk_gating_plan& pl, const LaunchEnv& env, const CUtensorMap& mx,
                         const CUtensorMap& mx64, const CUtensorMap& mw, int64_t T, int64_t H, int64_t E, int32_t k,
                         float* scores, int32_t* ids, const float* hscale, const float* gscale, float* logits,
                         cudaStream_t stream) {
  uint32_t* err = env.err_word;
  if (pl.variant == TK_VARIANT_FEW_TOKENS) {
    if constexpr (FP8) {
      return TK_ERR_UNSUPPORTED;  // the planner chooses it for bf16 inputs only
    } else {
      if (env.workspace == nullptr || env.hidden == nullptr || env.gate == nullptr) return TK_ERR_INVALID_ARG;
      if (env.route.table != nullptr) return TK_ERR_UNSUPPORTED;  // this kernel takes no routing counts
      FewTokenParams fp;
      fp.hidden = static_cast<const uint16_t*>(env.hidden);
      fp.gate = static_cast<const uint16_t*>(env.gate);
      fp.T = static_cast<int32_t>(T);
      fp.H = static_cast<int32_t>(H);
      fp.E = static_cast<int32_t>(E);
      fp.k = k;
      fp.e_blocks = pl.n_pad / FEW_EXPERTS;
      fp.h_blocks = pl.split_h;
      fp.h_rows = pl.h_rows;
      fp.e_pad = pl.n_pad;
      fp.counter = static_cast<uint32_t*>(env.workspace);
      fp.part = reinterpret_cast<float*>(static_cast<uint8_t*>(env.workspace) + FEW_COUNTER_BYTES);
      fp.scores = scores;
      fp.ids = ids;
      fp.logits = logits;
      fp.err_word = err;
      fp.timeout_ns = env.timeout_ns;
      fp.clock = env.clock;
      if (k <= 4) return launch_few_tokens<4>(pl, fp, stream);
      if (k <= 8) return launch_few_tokens<8>(pl, fp, stream);
      if (k <= 16) return launch_few_tokens<16>(pl, fp, stream);
      return launch_few_tokens<32>(pl, fp, stream);
    }
  }
  if (pl.variant == TK_VARIANT_SPLIT_H) {
    SplitHParams sp;
    sp.T = static_cast<int32_t>(T);
    sp.H = static_cast<int32_t>(H);
    sp.E = static_cast<int32_t>(E);
    sp.k = k;
    sp.n_pad = pl.n_pad;
    sp.e_groups = pl.expert_groups;
    sp.kps = pl.slices_per_stage;
    sp.num_tiles = pl.num_tiles;
    sp.k_blocks = pl.k_blocks;
    sp.stages = pl.stages;
    sp.b_boxes = (min_int(pl.n_pad, E_GROUP) + B_BOX_N - 1) / B_BOX_N;
    sp.row_stride = split_row_stride(E);
    sp.tmem_cols = static_cast<uint32_t>(pl.tmem_cols);
    sp.timeout_ns = env.timeout_ns;
    sp.scores = scores;
    sp.ids = ids;
    sp.err_word = err;
    sp.hscale = hscale;
    sp.gscale = gscale;
    sp.logits = logits;
    sp.clock = env.clock;
    sp.route = env.route;
    const int mc = env.max_split_cluster;
    // lists of 4 also serve k = 1, 2 (fewer kernel instances to build; an
    // insertion into 4 slots costs little more than into 1 or 2)
    if (k <= 4) return launch_split_h<4, FP8>(pl, mc, mx, mw, sp, stream);
    if (k <= 8) return launch_split_h<8, FP8>(pl, mc, mx, mw, sp, stream);
    if (k <= 16) return launch_split_h<16, FP8>(pl, mc, mx, mw, sp, stream);
    return launch_split_h<32, FP8>(pl, mc, mx, mw, sp, stream);
  }

  RowTileParams prm;
  prm.T = static_cast<int32_t>(T);
  prm.H = static_cast<int32_t>(H);
  prm.E = static_cast<int32_t>(E);
  prm.k = k;
  prm.n_pad = pl.n_pad;
  prm.e_groups = pl.expert_groups;
  prm.acc_stride = round_up(min_int(pl.n_pad, E_GROUP), 32);
  prm.acc_bufs = 2 * prm.acc_stride <= 512 ? 2 : 1;
  prm.num_tiles = pl.num_tiles;
  prm.num_half = pl.num_half_tiles;
  prm.k_blocks = pl.k_blocks;
  prm.stages = pl.stages;
  const int g_pad = min_int(pl.n_pad, E_GROUP);
  prm.b_boxes = pl.variant == TK_VARIANT_ROW_PAIRS ? g_pad / 2 / B_BOX_N : (g_pad + B_BOX_N - 1) / B_BOX_N;
  prm.tmem_cols = static_cast<uint32_t>(pl.tmem_cols);
  prm.timeout_ns = env.timeout_ns;
  prm.scores = scores;
  prm.ids = ids;
  prm.err_word = err;
  prm.hscale = hscale;
  prm.gscale = gscale;
  prm.logits = logits;
  prm.clock = env.clock;
  prm.route = env.route;
  prm.num_split = pl.num_split_tiles;
  prm.split_kb = pl.split_k_block;
  prm.part_cols = split_part_cols(E);
  prm.part_stride = split_part_stride(E);
  prm.split_token = env.split_token;
  prm.split_flags = nullptr;
  prm.split_part = nullptr;
  if (pl.num_split_tiles > 0) {
    if (env.workspace == nullptr) return TK_ERR_INVALID_ARG;
    prm.split_flags = static_cast<uint32_t*>(env.workspace);
    prm.split_part = reinterpret_cast<float*>(static_cast<uint8_t*>(env.workspace) +
                                              split_flag_bytes(pl.num_split_tiles));
  }

  if (k <= 4) return launch_row_variant<4, FP8>(pl, mx, mx64, mw, prm, stream);
  if (k <= 8) return launch_row_variant<8, FP8>(pl, mx, mx64, mw, prm, stream);
  if (k <= 16) return launch_row_variant<16, FP8>(pl, mx, mx64, mw, prm, stream);
  return launch_row_variant<32, FP8>(pl, mx, mx64, mw, prm, stream);
}

}  // namespace tkg
