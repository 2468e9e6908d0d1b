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
// position p = slot_pos[s] of this rank's expert-grouped order (offsets and
// slot_pos from tk_gating_route); its row in the expert buffer is
// rows[e] + (p - offsets[e]).  Both kernels work token by token, a warp per
// part of a token's row (EP_PART_VECS 16-byte vectors), over as many CTAs as
// the SMs hold at once.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace tkg {

constexpr int EP_THREADS = 256;  // 8 warps; a warp moves one row at a time

struct EpDispatchParams {
  const uint4* tokens;          // [T, H] bf16, rows of vec_per_row 16-byte vectors
  const int32_t* ids;           // [T * k]
  const int32_t* offsets;       // [E + 1]
  const int32_t* slot_pos;      // [T * k]
  const uint64_t* rows;         // [E] destination address of expert e's first row
  uint32_t* err_word;           // bit EP_ERR_ROW: a row address was not 16-byte aligned
  int64_t T;
  int64_t vec_per_row;          // H / 8
  int64_t part_vecs;            // 16-byte vectors of a row part (a multiple of 32, or the whole row)
  int32_t parts;                // parts per row
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
constexpr int EP_LANE_VECS = static_cast<int>(EP_PART_VECS / 32);  // a lane's vectors of one part, at most

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

// Row address of assignment s = t*k + lane for lane < k (0: nothing there --
// an id outside [0, E), slot_pos -1, a position outside its expert's range, or
// a row address that is not 16-byte aligned, which is also reported).
__device__ __forceinline__ uint64_t ep_row_of(const uint64_t* rows, const int32_t* ids, const int32_t* offsets,
                                              const int32_t* slot_pos, int64_t s, int32_t E, int64_t vec_per_row,
                                              uint32_t* err_word) {
  const int32_t e = __ldg(ids + s);
  const int32_t pos = __ldg(slot_pos + s);
  if (static_cast<uint32_t>(e) >= static_cast<uint32_t>(E) || pos < 0) return 0;
  const int32_t o0 = __ldg(offsets + e), o1 = __ldg(offsets + e + 1);
  const uint64_t base = __ldg(rows + e);
  if (pos < o0 || pos >= o1) return 0;
  if (base & 15u) {
    atomicOr(err_word, EP_ERR_ROW);
    return 0;
  }
  return base + static_cast<uint64_t>(pos - o0) * static_cast<uint64_t>(vec_per_row) * 16u;
}

// One warp per part of a token's row (grid-stride over T x parts work items):
// the token's vectors are loaded once and stored to each of its k destination
// rows (this rank's buffers or peers'), so a token row crosses from memory once
// however many experts it goes to.  Lane j < k looks up assignment j's row; the
// warp reads the addresses by shuffle.
template <int KMAX>
__global__ void __launch_bounds__(EP_THREADS) ep_dispatch_kernel(const EpDispatchParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * EP_THREADS + threadIdx.x) >> 5;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (EP_THREADS / 32);
  const int64_t items = p.T * p.parts;
  for (int64_t item = warp; item < items; item += warps) {
    const int64_t t = item / p.parts;
    const int64_t v0 = (item - t * p.parts) * p.part_vecs;
    const int64_t v1 = v0 + p.part_vecs < p.vec_per_row ? v0 + p.part_vecs : p.vec_per_row;
    const uint64_t my_row =
        lane < p.k ? ep_row_of(p.rows, p.ids, p.offsets, p.slot_pos, t * p.k + lane, p.E, p.vec_per_row, p.err_word)
                   : 0;
    uint64_t row[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) row[j] = __shfl_sync(0xffffffffu, my_row, j);
    // all of this lane's vectors of the part in flight at once, then each stored k times
    const uint4* src = p.tokens + t * p.vec_per_row;
    uint4 x[EP_LANE_VECS];
#pragma unroll
    for (int u = 0; u < EP_LANE_VECS; ++u)
      if (v0 + lane + 32 * u < v1) x[u] = ep_ld_nc(src + v0 + lane + 32 * u);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < p.k && row[j] != 0) {
        uint4* dst = reinterpret_cast<uint4*>(row[j]) + v0 + lane;
#pragma unroll
        for (int u = 0; u < EP_LANE_VECS; ++u)
          if (v0 + lane + 32 * u < v1) dst[32 * u] = x[u];
      }
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
      my_row = ep_row_of(p.rows, p.ids, p.offsets, p.slot_pos, s, p.E, p.vec_per_row, p.err_word);
      my_w = __ldg(p.scores + s);
    }
    uint64_t row[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      row[j] = __shfl_sync(0xffffffffu, my_row, j);
      w[j] = __shfl_sync(0xffffffffu, my_w, j);
    }
    uint4* dst = p.out + t * p.vec_per_row;
    // two of the lane's vectors per step: up to 2 x 8 row loads in flight
    for (int64_t v = v0 + lane; v < v1; v += 64) {
      const bool two = v + 32 < v1;
      float acc[2][8] = {{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}};
      constexpr int G = KMAX < 8 ? KMAX : 8;  // rows loaded before their multiply-adds
#pragma unroll
      for (int j0 = 0; j0 < KMAX; j0 += G) {
        uint4 y[2][G];
#pragma unroll
        for (int u = 0; u < G; ++u)
          if (j0 + u < p.k && row[j0 + u] != 0) {
            const uint4* r = reinterpret_cast<const uint4*>(row[j0 + u]);
            y[0][u] = ep_ld(r + v);
            if (two) y[1][u] = ep_ld(r + v + 32);
          }
#pragma unroll
        for (int u = 0; u < G; ++u)
          if (j0 + u < p.k && row[j0 + u] != 0) {
            ep_fma8(acc[0], w[j0 + u], y[0][u]);
            if (two) ep_fma8(acc[1], w[j0 + u], y[1][u]);
          }
      }
      dst[v] = make_uint4(ep_pack_bf16x2(acc[0][0], acc[0][1]), ep_pack_bf16x2(acc[0][2], acc[0][3]),
                          ep_pack_bf16x2(acc[0][4], acc[0][5]), ep_pack_bf16x2(acc[0][6], acc[0][7]));
      if (two)
        dst[v + 32] = make_uint4(ep_pack_bf16x2(acc[1][0], acc[1][1]), ep_pack_bf16x2(acc[1][2], acc[1][3]),
                                 ep_pack_bf16x2(acc[1][4], acc[1][5]), ep_pack_bf16x2(acc[1][6], acc[1][7]));
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
