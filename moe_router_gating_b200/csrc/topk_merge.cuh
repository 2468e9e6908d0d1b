// Merging per-thread top-k lists across the lanes of a warp.
//
// Each participating lane holds a list sorted under the total order
// (value descending, index ascending) -- the invariant RowTopK keeps.  Given two
// sorted lists a and b of length L, c_j = better(a_j, b_{L-1-j}) holds the best
// L entries of a U b as a bitonic sequence; a bitonic merge network (compare and
// exchange at distances L/2, L/4, ..., 1) then sorts it.  Repeating this with
// partners lane^1, lane^2, ... leaves every lane of a group of G lanes with the
// best L entries of the group.  Indices are distinct, so the order is strict
// and every lane ends with the same list.
#pragma once

#include <cstdint>

#include "topk_epilogue.cuh"

namespace tkg {

__device__ __forceinline__ bool ranks_before(float va, int32_t ia, float vb, int32_t ib) {
  return va > vb || (va == vb && ia < ib);
}

// t <- the best L entries of t U (bv, bi), sorted; (bv, bi) is a sorted list of L.
template <int L>
__device__ __forceinline__ void merge_sorted(RowTopK<L>& t, const float (&bv)[L], const int32_t (&bi)[L]) {
#pragma unroll
  for (int j = 0; j < L; ++j) {
    const bool take = ranks_before(bv[L - 1 - j], bi[L - 1 - j], t.v[j], t.i[j]);
    t.v[j] = take ? bv[L - 1 - j] : t.v[j];
    t.i[j] = take ? bi[L - 1 - j] : t.i[j];
  }
#pragma unroll
  for (int d = L / 2; d >= 1; d /= 2) {
#pragma unroll
    for (int j = 0; j < L; ++j) {
      if ((j & d) == 0) {
        const bool swap = ranks_before(t.v[j + d], t.i[j + d], t.v[j], t.i[j]);
        const float a = t.v[j], b = t.v[j + d];
        const int32_t ia = t.i[j], ib = t.i[j + d];
        t.v[j] = swap ? b : a;
        t.v[j + d] = swap ? a : b;
        t.i[j] = swap ? ib : ia;
        t.i[j + d] = swap ? ia : ib;
      }
    }
  }
}

template <int L>
__device__ __forceinline__ void merge_with_lane(RowTopK<L>& t, int lane_mask) {
  float pv[L];
  int32_t pi[L];
#pragma unroll
  for (int j = 0; j < L; ++j) {
    pv[j] = __shfl_xor_sync(0xffffffffu, t.v[j], lane_mask);
    pi[j] = __shfl_xor_sync(0xffffffffu, t.i[j], lane_mask);
  }
  merge_sorted(t, pv, pi);
}

// Merge the lists of groups of `group` consecutive lanes (a power of two <= 32).
// Every lane of the warp must call this with the same `group`.
template <int L>
__device__ __forceinline__ void merge_lane_groups(RowTopK<L>& t, int group) {
  for (int d = 1; d < group; d <<= 1) merge_with_lane(t, d);
}

}  // namespace tkg

namespace tkg {

// softmax_store by a group of >= k lanes that all hold the same sorted list:
// lane j (j < k, j = the lane's position in its group) computes exp(v_j - v_0),
// every lane gathers the k terms by shuffles and sums them in the order
// j = 0 .. k-1, and lane j stores entry j -- the arithmetic of
// RowTopK::softmax_store, spread over the lanes.  `store` is false for lanes
// whose group has no row to write (they still take part in the shuffles).
// Every lane of the warp must call this with the same `group` (>= k).
template <int L>
__device__ __forceinline__ void group_softmax_store(const RowTopK<L>& t, int k, int group, bool store,
                                                    float* __restrict__ score_row, int32_t* __restrict__ id_row) {
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int j = lane & (group - 1);
  const int base = lane - j;
  float vj = t.v[0];
  int32_t ij = t.i[0];
#pragma unroll
  for (int q = 1; q < L; ++q) {
    vj = q == j ? t.v[q] : vj;
    ij = q == j ? t.i[q] : ij;
  }
  const float ex = j < k ? expf(vj - t.v[0]) : 0.0f;
  float sum = 0.0f;
  for (int q = 0; q < L; ++q) {  // the same order as softmax_store
    const float e = __shfl_sync(0xffffffffu, ex, base + (q < group ? q : 0));
    sum += q < k ? e : 0.0f;
  }
  if (store && j < k) {
    score_row[j] = ex / sum;
    id_row[j] = ij;
  }
}

}  // namespace tkg
