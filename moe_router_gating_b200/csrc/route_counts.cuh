// Per-expert assignment counts taken by the gating kernels while they store
// their ids: the counting step of the routing metadata (chenxutan.com,
// "TileKernels 深度解析", section 4.2 "MoE Routing": dispatch groups the
// token-expert assignments by expert, which starts from how many assignments
// each expert received), moved into the gating epilogue so that the routing
// needs no pass of its own over the ids to count them.
//
// The table has one row per routing range (the slots [c*range_slots,
// (c+1)*range_slots) that CTA c of the placing kernel in route.cuh owns) and
// one column per expert: table[c][e] = the assignments s = t*k + j of range c
// whose expert is e.  Assignments are added one at a time (atomic adds in
// global memory, no returned value), so the table must be zero before the
// gating launch; the placing kernel reads it and leaves it zero again.
#pragma once

#include <cstdint>

#include "topk_epilogue.cuh"

namespace tkg {

struct RouteCounts {
  int32_t* table;        // [ranges][E4] int32; null: the launch does not count
  uint32_t range_slots;  // assignments per routing range (32 warps x L slots)
  int32_t E4;            // row pitch of the table (E rounded up to 4)
};

// Count assignment s (expert e) of the range that holds it; an id outside
// [0, E) is not counted (the placing kernel skips it the same way).  s < 2^31.
__device__ __forceinline__ void route_count_one(const RouteCounts& rc, uint32_t s, int32_t e, int32_t E) {
  if (static_cast<uint32_t>(e) < static_cast<uint32_t>(E))
    atomicAdd(rc.table + static_cast<int64_t>(s / rc.range_slots) * rc.E4 + e, 1);
}

// The k assignments of one row held by one thread (its sorted list).
template <int KMAX>
__device__ __forceinline__ void route_count_row(const RouteCounts& rc, const RowTopK<KMAX>& t, int k, int64_t row,
                                                int32_t E) {
  const uint32_t s0 = static_cast<uint32_t>(row) * static_cast<uint32_t>(k);
  // a row's k <= 32 assignments cross at most one range boundary (ranges hold
  // at least 4096): one division per row
  const uint32_t c0 = s0 / rc.range_slots;
  const uint32_t left = (c0 + 1) * rc.range_slots - s0;  // assignments of the row in range c0
  int32_t* r0 = rc.table + static_cast<int64_t>(c0) * rc.E4;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k && static_cast<uint32_t>(t.i[j]) < static_cast<uint32_t>(E))
      atomicAdd(r0 + (static_cast<uint32_t>(j) >= left ? rc.E4 : 0) + t.i[j], 1);
  }
}

// The same for a row whose list every lane of a group of `group` >= k lanes
// holds: lane j of the group counts entry j.  `active` is false for lanes
// whose group has no row.
template <int KMAX>
__device__ __forceinline__ void group_route_count(const RouteCounts& rc, const RowTopK<KMAX>& t, int k, int group,
                                                  bool active, int64_t row, int32_t E) {
  const int j = static_cast<int>(threadIdx.x & 31) & (group - 1);
  int32_t ij = t.i[0];
#pragma unroll
  for (int q = 1; q < KMAX; ++q) ij = q == j ? t.i[q] : ij;
  if (active && j < k)
    route_count_one(rc, static_cast<uint32_t>(row) * static_cast<uint32_t>(k) + static_cast<uint32_t>(j), ij, E);
}

}  // namespace tkg
