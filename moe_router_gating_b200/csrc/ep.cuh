// Expert-parallel dispatch and combine (chenxutan.com, "TileKernels 深度解析",
// section 4.2 "MoE Routing": fused_dispatch sends every token to the GPUs that
// hold the experts its expert_ids row names, fused_combine brings the experts'
// results back weighted by the gating scores; section 6 "DeepEP V2": the
// receiver pulls remote data instead of being pushed fine-grained messages).
//
// Both kernels address the expert buffers through a table of E row addresses,
// rows[e] = the first row of this source rank's block of expert e in the
// buffer of the rank that holds e -- a local address, or another GPU's memory
// mapped into this process.  The copy IS the exchange: dispatch stores each
// token row at its destination directly, and combine loads each expert
// output row from where it lies, so no staging copy and no separate
// all-to-all runs.  Plain 16-byte loads and stores; no multicast.
//
// Assignment s = t*k + j (token t, rank j) with expert e = ids[s] sits at
// position p = slot_pos[s] of this rank's expert-grouped order (offsets,
// sorted_slots, slot_pos from tk_gating_route); its row in the expert buffer
// is rows[e] + (p - offsets[e]).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace tkg {

constexpr int EP_THREADS = 256;  // 8 warps; a warp moves one row at a time
constexpr int EP_UNROLL = 4;     // 16-byte vectors in flight per lane

struct EpDispatchParams {
  const uint4* tokens;          // [T, H] bf16, rows of vec_per_row 16-byte vectors
  const int32_t* ids;           // [T * k]
  const int32_t* offsets;       // [E + 1]
  const int32_t* sorted_slots;  // [T * k]
  const uint64_t* rows;         // [E] destination address of expert e's first row
  uint32_t* err_word;           // bit EP_ERR_ROW: a row address was not 16-byte aligned
  int64_t vec_per_row;          // H / 8
  int32_t k;
  int32_t E;
};

struct EpCombineParams {
  const uint64_t* rows;      // [E] address of expert e's first output row
  const int32_t* ids;        // [T * k]
  const int32_t* offsets;    // [E + 1]
  const int32_t* slot_pos;   // [T * k]
  const float* scores;       // [T * k]
  uint4* out;                // [T, H] bf16
  uint32_t* err_word;
  int64_t T;
  int64_t vec_per_row;
  int64_t part_vecs;  // 16-byte vectors of a row part (a multiple of 32, or the whole row)
  int32_t parts;      // parts per row: a warp combines one part of one token's row at a time
  int32_t k;
  int32_t E;
};

// Row parts of about 224 vectors (seven per lane): enough work items to spread
// a few thousand tokens evenly over every resident warp.
constexpr int64_t EP_PART_VECS = 224;

constexpr uint32_t EP_ERR_ROW = 1u << 8;

__device__ __forceinline__ uint4 ep_ld_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ep_ld(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// One warp per placed position p (grid-stride): copy token sorted_slots[p] / k
// to its row in the destination buffer of expert ids[sorted_slots[p]].
__global__ void __launch_bounds__(EP_THREADS) ep_dispatch_kernel(const EpDispatchParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * EP_THREADS + threadIdx.x) >> 5;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (EP_THREADS / 32);
  const int64_t placed = __ldg(p.offsets + p.E);
  for (int64_t pos = warp; pos < placed; pos += warps) {
    const int32_t s = __ldg(p.sorted_slots + pos);
    const int32_t e = __ldg(p.ids + s);
    if (static_cast<uint32_t>(e) >= static_cast<uint32_t>(p.E)) continue;  // not produced by the routing
    const int32_t o0 = __ldg(p.offsets + e), o1 = __ldg(p.offsets + e + 1);
    if (pos < o0 || pos >= o1) continue;
    const uint64_t base = __ldg(p.rows + e);
    if (base & 15u) {
      if (lane == 0) atomicOr(p.err_word, EP_ERR_ROW);
      continue;
    }
    const uint4* src = p.tokens + static_cast<int64_t>(s / p.k) * p.vec_per_row;
    uint4* dst = reinterpret_cast<uint4*>(base) + (pos - o0) * p.vec_per_row;
    int64_t v = lane;
    for (; v + 32 * (EP_UNROLL - 1) < p.vec_per_row; v += 32 * EP_UNROLL) {
      uint4 r[EP_UNROLL];
#pragma unroll
      for (int u = 0; u < EP_UNROLL; ++u) r[u] = ep_ld_nc(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < EP_UNROLL; ++u) dst[v + 32 * u] = r[u];
    }
    for (; v < p.vec_per_row; v += 32) dst[v] = ep_ld_nc(src + v);
  }
  // the stores (possibly to another GPU) are ordered before whatever the host
  // orders after this kernel
  __threadfence_system();
}

__device__ __forceinline__ void ep_fma8(float (&acc)[8], float w, uint4 v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] = fmaf(w, __uint_as_float(u[q] << 16), acc[2 * q]);
    acc[2 * q + 1] = fmaf(w, __uint_as_float(u[q] & 0xffff0000u), acc[2 * q + 1]);
  }
}

__device__ __forceinline__ uint32_t ep_pack_bf16x2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

// One warp per part of a token's row (grid-stride over T x parts work items):
// out[t] = sum_{j < k} scores[t, j] * row(t, j), fp32 fused multiply-adds in
// rank order j = 0 .. k-1, rounded once to bf16.  Lane j < k looks up
// assignment j's row address; the warp reads them by shuffle.
template <int KMAX>
__global__ void __launch_bounds__(EP_THREADS) ep_combine_kernel(const EpCombineParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * EP_THREADS + threadIdx.x) >> 5;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (EP_THREADS / 32);
  const int64_t items = p.T * p.parts;
  for (int64_t item = warp; item < items; item += warps) {
    const int64_t t = item / p.parts;
    const int64_t v0 = (item - t * p.parts) * p.part_vecs;
    const int64_t v1 = v0 + p.part_vecs < p.vec_per_row ? v0 + p.part_vecs : p.vec_per_row;
    uint64_t my_row = 0;
    float my_w = 0.0f;
    if (lane < p.k) {
      const int64_t s = t * p.k + lane;
      const int32_t e = __ldg(p.ids + s);
      const int32_t pos = __ldg(p.slot_pos + s);
      if (static_cast<uint32_t>(e) < static_cast<uint32_t>(p.E) && pos >= 0) {
        const int32_t o0 = __ldg(p.offsets + e), o1 = __ldg(p.offsets + e + 1);
        const uint64_t base = __ldg(p.rows + e);
        if (pos >= o0 && pos < o1) {
          if (base & 15u)
            atomicOr(p.err_word, EP_ERR_ROW);
          else
            my_row = base + static_cast<uint64_t>(pos - o0) * static_cast<uint64_t>(p.vec_per_row) * 16u;
        }
        my_w = __ldg(p.scores + s);
      }
    }
    uint64_t row[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      row[j] = __shfl_sync(0xffffffffu, my_row, j);
      w[j] = __shfl_sync(0xffffffffu, my_w, j);
    }
    uint4* dst = p.out + t * p.vec_per_row;
    for (int64_t v = v0 + lane; v < v1; v += 32) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      constexpr int G = KMAX < 8 ? KMAX : 8;  // rows loaded before their multiply-adds
#pragma unroll
      for (int j0 = 0; j0 < KMAX; j0 += G) {
        uint4 y[G];
#pragma unroll
        for (int u = 0; u < G; ++u)
          if (j0 + u < p.k && row[j0 + u] != 0) y[u] = ep_ld(reinterpret_cast<const uint4*>(row[j0 + u]) + v);
#pragma unroll
        for (int u = 0; u < G; ++u)
          if (j0 + u < p.k && row[j0 + u] != 0) ep_fma8(acc, w[j0 + u], y[u]);
      }
      dst[v] = make_uint4(ep_pack_bf16x2(acc[0], acc[1]), ep_pack_bf16x2(acc[2], acc[3]),
                          ep_pack_bf16x2(acc[4], acc[5]), ep_pack_bf16x2(acc[6], acc[7]));
    }
  }
}

}  // namespace tkg

namespace tkg {

__device__ __forceinline__ int64_t ep_count(const int32_t* offsets_all, int s, int E, int e) {
  const int32_t* o = offsets_all + static_cast<int64_t>(s) * (E + 1);
  return static_cast<int64_t>(o[e + 1]) - o[e];
}

// The row-address tables of one source rank, from every rank's routing
// offsets (offsets_all[s * (E + 1) + e]: rank s's tk_gating_route offsets, so
// rank s has count(s, e) = offsets_all[s][e + 1] - offsets_all[s][e]
// assignments to expert e).  Rank q holds experts [q*per, (q+1)*per); its
// buffer lists them in ascending order, each expert's rows by source rank,
// ascending.  One CTA, thread e:
//   dest_row(e) = sum_{e' in [q*per, e)} total(e') + sum_{s < rank} count(s, e)
//   rows[e]     = bases[q] + dest_row(e) * row_bytes       (for every table)
//   recv_offsets[i] (i <= per) = the first row of this rank's i-th expert.
// Every index stays inside [0, R*(E+1)) and [0, E].
__global__ void __launch_bounds__(1024) ep_rows_table_kernel(const int32_t* offsets_all, int32_t R, int32_t E,
                                                             int32_t rank, const uint64_t* bases_a,
                                                             const uint64_t* bases_b, int64_t row_bytes,
                                                             uint64_t* rows_a, uint64_t* rows_b,
                                                             int32_t* recv_offsets) {
  __shared__ int64_t total[1024];
  const int per = E / R;
  const int e = threadIdx.x;
  if (e < E) {
    int64_t t = 0;
    for (int s = 0; s < R; ++s) t += ep_count(offsets_all, s, E, e);
    total[e] = t;
  }
  __syncthreads();
  if (e < E) {
    const int q = e / per;
    int64_t row = 0;
    for (int x = q * per; x < e; ++x) row += total[x];
    for (int s = 0; s < rank; ++s) row += ep_count(offsets_all, s, E, e);
    rows_a[e] = bases_a[q] + static_cast<uint64_t>(row * row_bytes);
    if (rows_b != nullptr) rows_b[e] = bases_b[q] + static_cast<uint64_t>(row * row_bytes);
  }
  if (recv_offsets != nullptr && (e < per || e == 0)) {
    // thread e < per: this rank's expert e starts there; thread 0 also writes the total
    const int upto = e < per ? e : per;
    int64_t row = 0;
    for (int x = rank * per; x < rank * per + upto; ++x) row += total[x];
    recv_offsets[upto] = static_cast<int32_t>(row);
    if (e == 0) {
      int64_t all = 0;
      for (int x = rank * per; x < rank * per + per; ++x) all += total[x];
      recv_offsets[per] = static_cast<int32_t>(all);
    }
  }
}

}  // namespace tkg
