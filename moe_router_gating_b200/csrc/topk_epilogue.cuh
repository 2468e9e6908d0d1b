// Register-resident top-k and softmax for one token row per thread.
//
// Selection follows the strict total order (logit descending, expert index
// ascending).  Values are offered in increasing expert index, so a strict ">"
// comparison keeps the lower index ahead of an equal later one; -0.0 and +0.0
// compare equal under IEEE comparison, as the order requires.
#pragma once

#include <cstdint>

namespace tkg {

template <int KMAX>
struct RowTopK {
  float v[KMAX];
  int32_t i[KMAX];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      v[j] = -__int_as_float(0x7f800000);  // -inf
      i[j] = 0x7fffffff;
    }
  }

  // Offer (value, index); indices must arrive in increasing order.
  //
  // Branch-free sorted insertion: with c_j = (value beats slot j), the new slot
  // j holds the old slot j when !c_j, the old slot j-1 when c_{j-1} (the list is
  // sorted, so c_{j-1} implies c_j), and the offered pair otherwise.  All slot
  // updates read the old list, so they are independent of one another, and no
  // lane of a warp ever waits on another lane's insertion.  The comparisons are
  // taken into one bit mask before any slot changes: written as an array of
  // bools, nvcc 12.9 for sm_100a was seen to build lists of 4 that held the
  // offered pair twice (the list's first comparison redone against the updated
  // slot 0), in some loop contexts only.
  __device__ __forceinline__ void offer(float value, int32_t index) {
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) c |= static_cast<uint32_t>(value > v[j]) << j;
#pragma unroll
    for (int j = KMAX - 1; j > 0; --j) {
      const bool cj = (c >> j) & 1u;
      const bool cp = (c >> (j - 1)) & 1u;
      v[j] = cj ? (cp ? v[j - 1] : value) : v[j];
      i[j] = cj ? (cp ? i[j - 1] : index) : i[j];
    }
    v[0] = (c & 1u) ? value : v[0];
    i[0] = (c & 1u) ? index : i[0];
  }

  // Offer a candidate whose index may be lower than ones already held (used when
  // merging lists): the full (value desc, index asc) comparison decides.
  __device__ __forceinline__ void offer_any(float value, int32_t index) {
    const bool enter = value > v[KMAX - 1] || (value == v[KMAX - 1] && index < i[KMAX - 1]);
    if (enter) {
      v[KMAX - 1] = value;
      i[KMAX - 1] = index;
#pragma unroll
      for (int j = KMAX - 1; j > 0; --j) {
        const bool up = v[j] > v[j - 1] || (v[j] == v[j - 1] && i[j] < i[j - 1]);
        const float tv = v[j];
        const int32_t ti = i[j];
        v[j] = up ? v[j - 1] : v[j];
        i[j] = up ? i[j - 1] : i[j];
        v[j - 1] = up ? tv : v[j - 1];
        i[j - 1] = up ? ti : i[j - 1];
      }
    }
  }

  // scores[j] = exp(v_j - v_0) / sum_{i<k} exp(v_i - v_0); writes k entries of
  // the row (16-byte vector stores when k % 4 == 0).
  __device__ __forceinline__ void softmax_store(int k, float* __restrict__ score_row,
                                                int32_t* __restrict__ id_row) const {
    const float m = v[0];
    float ex[KMAX];
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ex[j] = (j < k) ? expf(v[j] - m) : 0.0f;
      sum += ex[j];
    }
    if constexpr (KMAX >= 4) {
      if ((k & 3) == 0) {
#pragma unroll
        for (int j = 0; j < KMAX; j += 4) {
          if (j < k) {
            *reinterpret_cast<float4*>(score_row + j) =
                make_float4(ex[j] / sum, ex[j + 1] / sum, ex[j + 2] / sum, ex[j + 3] / sum);
            *reinterpret_cast<int4*>(id_row + j) = make_int4(i[j], i[j + 1], i[j + 2], i[j + 3]);
          }
        }
        return;
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        score_row[j] = ex[j] / sum;
        id_row[j] = i[j];
      }
    }
  }
};

}  // namespace tkg
