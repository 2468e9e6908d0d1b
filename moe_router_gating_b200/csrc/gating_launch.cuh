// Launch interface of the fused gating kernels, shared by the host entry points
// (tk_gating.cu) and the two translation units that instantiate the kernels
// (gating_bf16.cu, gating_fp8.cu; the definitions are in gating_launch_impl.cuh).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tk_gating.h"
#include "gating_row_tiles.cuh"
#include "gating_split_h.cuh"
#include "gating_few_tokens.cuh"

namespace tkg {

constexpr int kMaxDynamicSmem = 232448;  // 227 KB opt-in per CTA on sm_100

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Floats per staged partial row of the split-H exchange (one pass of up to 256
// experts; +4 spreads the rows over the shared-memory banks).
inline int split_row_stride(int64_t E) { return round_up(static_cast<int>(E < N_CHUNK ? E : N_CHUNK), 32) + 4; }

// What a launch needs from the device state.
struct LaunchEnv {
  int max_split_cluster;  // largest split-H cluster the device co-schedules
  uint32_t* err_word;     // device error word of the bounded waits
  uint64_t timeout_ns;    // bounded-wait limit
  uint64_t* clock;        // SM-clock counters of the launches (cycles, ns, launches)
  RouteCounts route;      // per-expert counts of the stored ids by routing range; table null: none
  void* workspace;        // split last round (plan.num_split_tiles > 0): flags, then first-half partials;
                          // few-token variant: its counter, then the CTAs' partial logits
  uint32_t split_token;   // non-zero, different for every launch
  const void* hidden;     // the inputs themselves: the few-token kernel reads them with plain loads
  const void* gate;
};

// Workspace of the few-token variant: the arrival counter (then padding to 256
// bytes) and the CTAs' partial logits, h_blocks x T rows of n_pad floats.
constexpr int64_t FEW_COUNTER_BYTES = 256;
inline int64_t few_token_workspace_bytes(int64_t T, int h_blocks, int e_pad) {
  return FEW_COUNTER_BYTES + static_cast<int64_t>(h_blocks) * T * e_pad * 4;
}

// Workspace of a split last round: num_split x 2 uint32 flags (8 bytes per tile,
// rounded up to 256), then the first halves' fp32 rows, num_split x 256 rows of
// round_up(E, 32) + 4 floats (the 4 keep consecutive rows off the same
// shared-memory banks once copied there).
inline int split_part_cols(int64_t E) { return round_up(static_cast<int>(E), 32); }
inline int split_part_stride(int64_t E) { return split_part_cols(E) + 4; }
inline int64_t split_flag_bytes(int num_split) { return (static_cast<int64_t>(num_split) * 8 + 255) / 256 * 256; }
inline int64_t split_workspace_bytes(int num_split, int64_t E) {
  return num_split > 0
             ? split_flag_bytes(num_split) + static_cast<int64_t>(num_split) * 256 * split_part_stride(E) * 4
             : 0;
}

// Shared-memory limits (and non-portable cluster sizes) of every kernel instance
// of one precision; once per device.
template <bool FP8>
bool set_up_gating_kernels();

// Launch the planned kernel on encoded maps.  FP8: hscale / gscale are the
// per-token and per-expert scales (unused for bf16).  logits: optional fp32
// [T, E] that also receives every logit the selection ranks (verification).
template <bool FP8>
tk_status launch_planned(const tk_gating_plan& pl, const LaunchEnv& env, const CUtensorMap& mx,
                         const CUtensorMap& mx64, const CUtensorMap& mw, int64_t T, int64_t H, int64_t E, int32_t k,
                         float* scores, int32_t* ids, const float* hscale, const float* gscale, float* logits,
                         cudaStream_t stream);

extern template bool set_up_gating_kernels<false>();
extern template bool set_up_gating_kernels<true>();
extern template tk_status launch_planned<false>(const tk_gating_plan&, const LaunchEnv&, const CUtensorMap&,
                                                const CUtensorMap&, const CUtensorMap&, int64_t, int64_t, int64_t,
                                                int32_t, float*, int32_t*, const float*, const float*, float*,
                                                cudaStream_t);
extern template tk_status launch_planned<true>(const tk_gating_plan&, const LaunchEnv&, const CUtensorMap&,
                                               const CUtensorMap&, const CUtensorMap&, int64_t, int64_t, int64_t,
                                               int32_t, float*, int32_t*, const float*, const float*, float*,
                                               cudaStream_t);

// Clusters of 2, 4, 8 and 16 full-shared-memory split-H CTAs that the current
// device runs at once, into counts[0..3] (0 where a size cannot run).
void measure_split_cluster_capacity(int counts[4]);

}  // namespace tkg
