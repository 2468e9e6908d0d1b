// Routing metadata of MoE dispatch, local part: the token-expert assignments
// ids[T, k] grouped by expert (chenxutan.com, "TileKernels 深度解析", section
// 4.2 "MoE Routing": dispatch sends each token to the experts its expert_ids
// row names and hands combine the indices that put the results back).
//
// For the n = T*k assignments s = t*k + j with expert e = ids[s] (valid when
// 0 <= e < E), the outputs are
//   offsets[e]      assignments to experts < e (exclusive prefix sum; offsets[E]
//                   = assignments placed),
//   sorted_slots[p] the assignment at position p of the expert-grouped order, in
//                   ascending s inside an expert (a stable order, so unique),
//   slot_pos[s]     its position p (the inverse permutation; -1 for an invalid
//                   id, which is neither counted nor placed).
//
// Every slot belongs to exactly one warp range: warp w of CTA c owns
// [(c*W + w)*L, (c*W + w + 1)*L) clipped to n, with L a multiple of 32.  The
// position of slot s with expert e is
//   offsets[e] + (slots of e in earlier CTAs) + (in earlier warps of its CTA)
//              + (in earlier 32-slot batches of its warp) + (in lower lanes of
//              its batch),
// the last term from ballots over the bits of e (route_group_mask).
//
// One CTA (n <= W*L): route_scatter_kernel<NB, true> alone, no workspace.
// More CTAs: route_count_kernel writes each CTA's per-expert counts into the
// workspace counts[G][E4]; route_scatter_kernel<NB, false>, launched as a
// programmatic dependent of it, recounts its own range per warp while the
// counts drain, then reads the whole table (its CTA prefix and the totals).
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace tkg {

constexpr int ROUTE_WARPS = 32;
constexpr int ROUTE_THREADS = ROUTE_WARPS * 32;
constexpr int ROUTE_MIN_WARP_SLOTS = 128;  // at least four 32-slot batches per warp
constexpr int ROUTE_PREFETCH = 8;          // batches of ids in flight per warp

// Where the placing kernel gets the per-CTA counts from.
enum RouteMode : int {
  ROUTE_ONE_CTA = 0,  // one CTA: it counts its own slots, no table
  ROUTE_TABLE = 1,    // route_count_kernel wrote the table just before
  ROUTE_FUSED = 2,    // the gating kernel added its ids to the table (route_counts.cuh)
};

struct RouteParams {
  const int32_t* ids;
  int64_t n;             // T * k
  int32_t E;
  int32_t E4;            // row pitch of counts (E rounded up to 4)
  int32_t Ep;            // row pitch of the per-warp shared-memory counts (E + 1: conflict-free columns)
  int32_t G;             // CTAs
  int64_t warp_slots;    // L: slots per warp range, a multiple of 32
  int32_t* counts;       // workspace [G][E4] (several CTAs only)
  uint32_t* done;        // ROUTE_FUSED: CTAs that have read the table (zero between calls)
  int32_t* offsets;      // [E + 1]
  int32_t* sorted_slots; // [n]
  int32_t* slot_pos;     // [n]
  uint32_t* err_word;    // device error word (debug-build index checks)
};

__device__ __forceinline__ uint32_t route_lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Expert of slot s, or -1 when s is past the range or the id is out of [0, E).
__device__ __forceinline__ int32_t route_expert(const int32_t* ids, int64_t s, int64_t end, int32_t E) {
  const int32_t e = s < end ? __ldg(ids + s) : -1;
  return static_cast<uint32_t>(e) < static_cast<uint32_t>(E) ? e : -1;
}

// The lanes of the warp whose expert equals this lane's (-1 lanes form their
// own group): one ballot per bit of the expert index (NB >= bits of E - 1)
// plus one for validity.
template <int NB>
__device__ __forceinline__ uint32_t route_group_mask(int32_t e) {
  const uint32_t valid = __ballot_sync(0xffffffffu, e >= 0);
  uint32_t m = e >= 0 ? valid : ~valid;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint32_t flip = ((e >> b) & 1) ? 0u : 0xffffffffu;
    m &= __ballot_sync(0xffffffffu, (e >> b) & 1) ^ flip;
  }
  return m;
}

__device__ __forceinline__ void route_warp_range(const RouteParams& p, int64_t* beg, int64_t* end) {
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * ROUTE_WARPS + (threadIdx.x >> 5);
  const int64_t b = gw * p.warp_slots;
  *beg = b < p.n ? b : p.n;
  *end = b + p.warp_slots < p.n ? b + p.warp_slots : p.n;
}

// Per-warp counts of this CTA's slots: hist[w * Ep + e] (shared memory, zeroed
// here).  Ends with a CTA barrier.
__device__ __forceinline__ void route_cta_warp_counts(const RouteParams& p, int32_t* hist, int64_t beg,
                                                      int64_t end) {
  for (int i = threadIdx.x; i < ROUTE_WARPS * p.Ep; i += ROUTE_THREADS) hist[i] = 0;
  __syncthreads();
  int32_t* row = hist + (threadIdx.x >> 5) * p.Ep;
  const uint32_t lane = threadIdx.x & 31u;
  for (int64_t b0 = beg; b0 < end; b0 += 32 * ROUTE_PREFETCH) {
    int32_t e[ROUTE_PREFETCH];
#pragma unroll
    for (int i = 0; i < ROUTE_PREFETCH; ++i) e[i] = route_expert(p.ids, b0 + i * 32 + lane, end, p.E);
#pragma unroll
    for (int i = 0; i < ROUTE_PREFETCH; ++i)
      if (e[i] >= 0) atomicAdd(row + e[i], 1);
  }
  __syncthreads();
}

// Dynamic shared memory: hist[ROUTE_WARPS][Ep] int32.
__global__ void __launch_bounds__(ROUTE_THREADS) route_count_kernel(const RouteParams p) {
  // launched as a programmatic dependent of whatever precedes it (the gating
  // kernel, typically): the ids are complete and visible past this wait
  pdl_wait_primary();
  pdl_launch_dependents();  // the scatter kernel may start its own recount now
  extern __shared__ int32_t route_smem[];
  int64_t beg, end;
  route_warp_range(p, &beg, &end);
  route_cta_warp_counts(p, route_smem, beg, end);
  int32_t* row = p.counts + static_cast<int64_t>(blockIdx.x) * p.E4;
  for (int e = threadIdx.x; e < p.E4; e += ROUTE_THREADS) {
    int32_t c = 0;
    if (e < p.E) {
#pragma unroll 8
      for (int w = 0; w < ROUTE_WARPS; ++w) c += route_smem[w * p.Ep + e];
    }
    row[e] = c;
  }
}

// Exclusive prefix sum of v[0..E) in place, by the whole CTA; returns the total.
// Each thread takes a run of `per` consecutive entries.
__device__ __forceinline__ int32_t route_block_exclusive_scan(int32_t* v, int32_t E, int32_t* warp_sums) {
  const int per = (E + ROUTE_THREADS - 1) / ROUTE_THREADS;
  const int lo = threadIdx.x * per;
  const int hi = lo + per < E ? lo + per : E;
  int32_t local = 0;
  for (int e = lo; e < hi; ++e) local += v[e];
  const uint32_t lane = threadIdx.x & 31u;
  int32_t incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t up = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= static_cast<uint32_t>(d)) incl += up;
  }
  if (lane == 31) warp_sums[threadIdx.x >> 5] = incl;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int32_t ws = threadIdx.x < ROUTE_WARPS ? warp_sums[threadIdx.x] : 0;
    int32_t wincl = ws;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t up = __shfl_up_sync(0xffffffffu, wincl, d);
      if (lane >= static_cast<uint32_t>(d)) wincl += up;
    }
    if (threadIdx.x < ROUTE_WARPS) warp_sums[threadIdx.x] = wincl - ws;  // exclusive per warp
    if (threadIdx.x == ROUTE_WARPS - 1) warp_sums[ROUTE_WARPS] = wincl;  // total
  }
  __syncthreads();
  int32_t run = warp_sums[threadIdx.x >> 5] + incl - local;
  for (int e = lo; e < hi; ++e) {
    const int32_t c = v[e];
    v[e] = run;
    run += c;
  }
  const int32_t total = warp_sums[ROUTE_WARPS];
  __syncthreads();
  return total;
}

// Column sums of the counts table: total[e] over all CTAs, below[e] over the
// CTAs before this one.  `part` holds 2 * ROUTE_THREADS int4 of scratch.
// own_row (optional, E4 words of shared memory) receives this CTA's own row of
// the table as it goes by.
__device__ __forceinline__ void route_table_sums(const RouteParams& p, int32_t* total, int32_t* below,
                                                 int4* part, int32_t* own_row = nullptr) {
  const int quads = p.E4 / 4;
  const int groups = ROUTE_THREADS / quads;  // row groups (quads <= ROUTE_THREADS)
  const int q = threadIdx.x % quads;
  const int r0 = threadIdx.x / quads;
  int4 sa = make_int4(0, 0, 0, 0), sb = make_int4(0, 0, 0, 0);
  if (r0 < groups) {
    const int4* tab = reinterpret_cast<const int4*>(p.counts);
    constexpr int U = 8;  // independent 16-byte loads in flight per thread
    for (int r = r0; r < p.G; r += U * groups) {
      int4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int rr = r + u * groups;
        v[u] = rr < p.G ? __ldcg(tab + static_cast<int64_t>(rr) * quads + q) : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (own_row != nullptr && r + u * groups == static_cast<int>(blockIdx.x))
          reinterpret_cast<int4*>(own_row)[q] = v[u];
        sa.x += v[u].x; sa.y += v[u].y; sa.z += v[u].z; sa.w += v[u].w;
        if (r + u * groups < static_cast<int>(blockIdx.x)) {
          sb.x += v[u].x; sb.y += v[u].y; sb.z += v[u].z; sb.w += v[u].w;
        }
      }
    }
  }
  int4* part_all = part;
  int4* part_below = part + ROUTE_THREADS;
  part_all[threadIdx.x] = sa;
  part_below[threadIdx.x] = sb;
  __syncthreads();
  for (int e = threadIdx.x; e < p.E4; e += ROUTE_THREADS) {
    const int qq = e >> 2, comp = e & 3;
    int32_t a = 0, b = 0;
    for (int g = 0; g < groups; ++g) {
      a += reinterpret_cast<const int32_t*>(part_all + g * quads + qq)[comp];
      b += reinterpret_cast<const int32_t*>(part_below + g * quads + qq)[comp];
    }
    total[e] = e < p.E ? a : 0;
    below[e] = b;
  }
  __syncthreads();
}

// Dynamic shared memory layout (int32 words):
//   base  [ROUTE_WARPS][Ep]  per-warp counts, then per-warp running positions
//   total [E4]               counts over all CTAs, then the global offsets
//   below [E4]               counts over CTAs before this one
//   part  [2][ROUTE_THREADS] int4 partial column sums (several CTAs only)
//   warp_sums [ROUTE_WARPS + 1]
template <int NB, int MODE>
__global__ void __launch_bounds__(ROUTE_THREADS) route_scatter_kernel(const RouteParams p) {
  extern __shared__ int32_t route_smem[];
  int32_t* base = route_smem;
  int32_t* total = base + ROUTE_WARPS * p.Ep;
  int32_t* below = total + p.E4;
  int32_t* warp_sums = below + p.E4;
  int4* part = reinterpret_cast<int4*>(warp_sums + 36);  // 16-byte aligned: Ep*32 + 2*E4 + 36 is a multiple of 4
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31u;
  __shared__ int route_flags[2];  // [0] this CTA's table row disagrees with its ids, [1] this CTA read the table last
  // counts from the gating: this CTA's row of the table, kept from the column sums' pass
  __shared__ __align__(16) int32_t own_row[MODE == ROUTE_FUSED ? TK_ROUTE_MAX_EXPERTS : 4];

  // 1. this CTA's per-warp counts.  One CTA, or counts from the gating: this
  //    kernel is the programmatic dependent of the kernel that wrote the ids (and
  //    the table) and waits for it first.  Counts from route_count_kernel: that
  //    kernel let this one start only after its own wait, so the ids are complete
  //    and may be read before this kernel's dependency wait.
  if (MODE != ROUTE_TABLE) pdl_wait_primary();
  int64_t beg, end;
  route_warp_range(p, &beg, &end);
  route_cta_warp_counts(p, base, beg, end);

  // 2. per-expert totals and the counts of earlier CTAs
  if (MODE == ROUTE_ONE_CTA) {
    for (int e = threadIdx.x; e < p.E4; e += ROUTE_THREADS) {
      int32_t c = 0;
      if (e < p.E) {
#pragma unroll 8
        for (int w = 0; w < ROUTE_WARPS; ++w) c += base[w * p.Ep + e];
      }
      total[e] = c;
      below[e] = 0;
    }
    __syncthreads();
  } else {
    if (MODE == ROUTE_TABLE) pdl_wait_primary();  // the counts table is complete and visible
    if (MODE == ROUTE_FUSED && threadIdx.x == 0) route_flags[0] = 0;
    route_table_sums(p, total, below, part, MODE == ROUTE_FUSED ? own_row : nullptr);
    if (MODE == ROUTE_FUSED) {
      // every read of the table by this CTA is complete (route_table_sums ends
      // with a CTA barrier): count the arrival; the CTA that arrives last zeroes
      // the table right after the scan below (its fence here orders those stores
      // after every other CTA's reads, which preceded their arrivals)
      if (threadIdx.x == 0) {
        __threadfence();
        const bool last = atomicAdd(p.done, 1u) == static_cast<uint32_t>(p.G - 1);
        if (last) __threadfence();
        route_flags[1] = last;
      }
      // the gating's row of this CTA must equal what the CTA has just counted;
      // it does unless the table was not zero before the gating launch
      bool bad = false;
      for (int e = threadIdx.x; e < p.E; e += ROUTE_THREADS) {
        int32_t c = 0;
#pragma unroll 8
        for (int w = 0; w < ROUTE_WARPS; ++w) c += base[w * p.Ep + e];
        bad |= own_row[e] != c;
      }
      if (bad) route_flags[0] = 1;
    }
  }

  // 3. global offsets (every CTA forms them; CTA 0 stores them)
  const int32_t placed = route_block_exclusive_scan(total, p.E, warp_sums);  // (its barriers also publish route_flags)
  if (MODE == ROUTE_FUSED) {
    if (threadIdx.x == 0 && route_flags[0] != 0) atomicOr(p.err_word, ERR_ROUTE_COUNTS);
    // every CTA has read the table: the last one to arrive leaves it zero for the
    // next call (while the other CTAs place their slots)
    if (route_flags[1]) {
      int4* tab = reinterpret_cast<int4*>(p.counts);
      const int64_t quads = static_cast<int64_t>(p.G) * (p.E4 / 4);
      for (int64_t q = threadIdx.x; q < quads; q += ROUTE_THREADS) tab[q] = make_int4(0, 0, 0, 0);
      if (threadIdx.x == 0) *p.done = 0u;
    }
  }
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < p.E; e += ROUTE_THREADS) p.offsets[e] = total[e];
    if (threadIdx.x == 0) p.offsets[p.E] = placed;
  }

  // 4. each warp's first position per expert: offset + earlier CTAs + earlier
  //    warps (a warp-wide scan down the column of expert e, lane = warp index)
  for (int e = warp; e < p.E; e += ROUTE_WARPS) {
    const int32_t c = base[lane * p.Ep + e];
    int32_t incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t up = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= static_cast<uint32_t>(d)) incl += up;
    }
    base[lane * p.Ep + e] = total[e] + below[e] + incl - c;
  }
  __syncthreads();

  // 5. place this warp's slots in ascending order
  int32_t* my = base + warp * p.Ep;
  const uint32_t lt = route_lanemask_lt();
  for (int64_t b0 = beg; b0 < end; b0 += 32 * ROUTE_PREFETCH) {
    int32_t e[ROUTE_PREFETCH];
#pragma unroll
    for (int i = 0; i < ROUTE_PREFETCH; ++i) e[i] = route_expert(p.ids, b0 + i * 32 + lane, end, p.E);
#pragma unroll
    for (int i = 0; i < ROUTE_PREFETCH; ++i) {
      if (b0 + i * 32 >= end) break;  // warp-uniform
      const int64_t s = b0 + i * 32 + lane;
      const uint32_t grp = route_group_mask<NB>(e[i]);
      const int32_t pos = e[i] >= 0 ? my[e[i]] + __popc(grp & lt) : -1;
      __syncwarp();
      // the lowest lane of each group moves its expert's position past the group
      if (e[i] >= 0 && (grp & lt) == 0) my[e[i]] += __popc(grp);
      __syncwarp();
      // counts from the gating are checked, not trusted: a position outside
      // [0, n) is never written (ERR_ROUTE_COUNTS is set then)
      const bool in_range = MODE == ROUTE_FUSED ? pos < p.n : TK_CHECK(pos < p.n, p.err_word);
      if (s < end && in_range) {
        p.slot_pos[s] = pos;
        if (pos >= 0) p.sorted_slots[pos] = static_cast<int32_t>(s);
      }
    }
  }
}

}  // namespace tkg
