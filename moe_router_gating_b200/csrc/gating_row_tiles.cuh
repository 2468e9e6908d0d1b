// Persistent fused gating kernel over whole token tiles.
//
// Per tile: logits[rows, E] = hidden[rows, H] x gate[H, E] on the tensor cores
// (tcgen05.mma, bf16 in, fp32 accumulate in tensor memory), then per row top-k
// and softmax in registers; only scores and ids reach global memory.
//
// CG = 1: one CTA per 128-token tile (M = 128, N = E rounded up to 16).
// CG = 2: a CTA pair (cluster of 2) per 256-token tile, tcgen05 cta_group::2
//   (M = 256, N = 128 or 256).  Each CTA stages its own 128 hidden rows and half
//   of the gate columns; the leader (cluster rank 0) issues the MMAs, which read
//   both CTAs' shared memory and write each CTA's 128 rows x N logits into its
//   own tensor memory.  Per CTA this halves the gate bytes each tile pulls from
//   L2 compared with CG = 1.
//   More than 256 experts (up to 512): the MMA N is split into chunks of at
//   most 256 columns, one tcgen05.mma per chunk and K step, chunk c
//   accumulating experts [256c, 256c + N_c) in tensor-memory columns from 256c;
//   in a pair each CTA holds half of every chunk's gate columns.  The
//   accumulator then fills tensor memory, so it is single-buffered.
//   More than 512 experts (up to 1024): the experts form two groups of at most
//   512, and every tile is two work items, one per group, back to back on the
//   same CTA (pair); the epilogue keeps its rows' top-k lists across the two
//   items and stores after the second.  The hidden tile is streamed once per
//   group.
//   FP8 (E4M3) inputs (FP8 = true): the same kernel with tcgen05.mma
//   kind::f8f6f4 (K = 32 per instruction); a 128-byte swizzle row holds 128
//   K values instead of 64, so a K slice covers 128 elements of H with the
//   same shared-memory footprint.  The gate is expert-major [E, H] (K-major,
//   like the hidden rows); the epilogue multiplies each logit by its token's
//   and its expert's scale before the selection.
//   Balanced tail: when the last round of 256-token tiles would leave pairs
//   idle, the remaining rows run as 128-token "half" tiles (M = 128 pair MMAs,
//   64 rows per CTA): half the MMA cycles and three quarters of the bytes of a
//   full tile (each CTA still streams its whole gate half), measured at about
//   90% of a full tile's time.  A half-tile accumulator is folded in tensor
//   memory: lanes 0..63 hold the CTA's 64 rows for experts [0, N/2) and lanes
//   64..127 the same rows for experts [N/2, N).
//
// Warp roles (192 threads per CTA):
//   warp 0      TMA producer: 64-wide K slices of the hidden rows (K-major,
//               128-byte swizzle) and of the gate (MN-major, 128-byte swizzle,
//               64-expert boxes); a ring stage holds KB_PER_STAGE consecutive
//               slices.
//   warp 1      allocates tensor memory; in the (leader) CTA one lane issues
//               tcgen05.mma (4 per K slice, K = 16 each) and the commits that
//               free ring stages and publish finished accumulators.  Two slices
//               per stage halve the per-MMA cost of the ring's waits and commits
//               (measured ~15% faster than one slice per stage on the 65536-token
//               workload).
//   warps 2..5  epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 (one token row
//   (or 2..9)   per thread), keeps a running top-k, applies the softmax and
//               stores.  With eight epilogue warps (epi_warps), warps 2..5 take
//               the first half of a tile's expert columns and warps 6..9 the
//               second; the second half's lists go through shared memory to the
//               first half's threads, which merge them before the softmax.  The
//               accumulator is double-buffered in tensor memory, so the epilogue
//               of one tile overlaps the MMAs of the next.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "topk_epilogue.cuh"
#include "route_counts.cuh"
#include "topk_merge.cuh"

namespace tkg {

constexpr int BLOCK_M = 128;                            // token rows per CTA = TMEM lanes
constexpr int BLOCK_K = 64;                             // bf16 per 128-byte swizzle row
constexpr int UMMA_K = 16;                              // K per tcgen05.mma (kind::f16)
constexpr int A_STAGE_BYTES = BLOCK_M * BLOCK_K * 2;    // 16 KB hidden slice
constexpr int B_BOX_N = 64;                             // experts per gate box
constexpr int B_BOX_BYTES = BLOCK_K * B_BOX_N * 2;      // 8 KB gate box
constexpr int EPI_BARRIER_RESERVE = 256;                // barriers and flags after the ring (bytes)
constexpr int KB_PER_STAGE = 2;                         // 64-wide K slices per ring stage

// Epilogue warps of a kernel instance: one per tensor-memory lane quadrant, or
// two (each taking half of a tile's expert columns) where the selection is the
// larger cost -- lists of 16 or 32, or two expert groups per tile.  Measured on
// one B200 (outputs bitwise equal): 65536 x 2048 x 256 with k = 16 92.8 vs 111.6
// us, 20000 x 2048 x 512 FP8 with k = 32 140 vs 196 us, 20000 x 2048 x 1024 with
// k = 8 122-127 vs 129-140 us; with k <= 8 and one group no gain (train shape
// 199.7-204.6 vs 198.7-201.3 us), so those keep four.
__host__ __device__ constexpr int epi_warps(int kmax, int expert_groups) {
  return (kmax >= 16 || expert_groups == 2) ? 8 : 4;
}
__host__ __device__ constexpr int row_tile_threads(int kmax, int expert_groups) {
  return 64 + 32 * epi_warps(kmax, expert_groups);
}

constexpr int N_CHUNK = 256;                            // MMA N per instruction (chunk of experts)
constexpr int XPOSE_STRIDE = 36;                        // floats per row of a warp's 32 x 32 store tile (16-byte rows)

struct RowTileParams {
  int32_t T, H, E, k;
  int32_t n_pad;        // total MMA N over all experts (CG=1: E rounded up to 16; CG=2: a multiple of 128)
  int32_t e_groups;     // expert groups of at most 512 (1 or 2; the kernel's EG); group g from expert 512 g
  int32_t acc_stride;   // TMEM columns between accumulator buffers
  int32_t acc_bufs;     // accumulator buffers in TMEM (2, or 1 when n_pad > 256)
  int32_t num_tiles;    // full tiles of BLOCK_M * CG rows, starting at row 0
  int32_t num_half;     // pairs only: half tiles of BLOCK_M rows after the full tiles
  int32_t k_blocks;
  int32_t stages;       // ring stages of KB_PER_STAGE K slices
  int32_t b_boxes;      // gate boxes per K slice and CTA in the ring (group 0's count, the largest)
  uint32_t tmem_cols;
  uint64_t timeout_ns;
  float* scores;
  int32_t* ids;
  uint32_t* err_word;
  const float* hscale;  // FP8 only: per-token scales [T]
  const float* gscale;  // FP8 only: per-expert scales [E]
  float* logits;        // optional [T, E]: every logit the selection ranks is also stored (verification)
  uint64_t* clock;      // SM-clock counters: the first CTA adds its cycles and ns (and 1) per launch
  RouteCounts route;    // optional per-expert counts of the stored ids by routing range (route_counts.cuh)
  // Split last round (pairs with one expert group and four epilogue warps, the
  // workspace entry points): instead of half tiles, num_split 256-token tiles
  // after the full ones, each cut in H at K slice split_kb between two pairs.
  // Pair 2j ("first half") accumulates slices [0, split_kb) of split tile j and
  // stores its fp32 accumulator rows to split_part[j][256 rows][part_stride], then
  // sets split_flags[2j + CTA rank] = split_token; pair 2j + 1 accumulates the
  // rest, waits for that flag, adds the stored partial to its own (first half +
  // second half) and selects; it then clears the flag.
  int32_t num_split;
  int32_t split_kb;
  int32_t part_cols;      // E rounded up to 32
  int32_t part_stride;    // floats between stored rows: part_cols + 4 (rows 16 bytes off the banks' period)
  uint32_t split_token;   // non-zero, different for every launch
  float* split_part;
  uint32_t* split_flags;
};

// K elements of H per K slice: one 128-byte swizzle row of bf16 or of FP8 values.
template <bool FP8>
constexpr int slice_k() {
  return FP8 ? 128 : 64;
}

// Gate descriptor of K step kk (0..3) of a slice: bf16 gate MN-major (see
// b_desc_k_slice); FP8 gate K-major like the hidden rows (rows of 128 B, 8-row
// groups 1024 B apart, the 32-element K step 32 B into each row).
template <bool FP8>
__device__ __forceinline__ uint64_t gate_desc_k_slice(uint32_t b_addr, int kk);

template <bool FP8>
__host__ __device__ constexpr uint32_t mma_idesc(uint32_t m, uint32_t n) {
  return FP8 ? idesc_e4m3_f32(m, n) : idesc_bf16_f32(m, n, false, true);
}

// FP8: logit = accumulator * expert scale * token scale, for the 32 columns of
// a chunk (experts e0 .. e0+31); columns past E keep a finite product of the
// last scale and are skipped by the offer.
template <bool FP8>
__device__ __forceinline__ void scale_chunk(uint32_t (&r)[32], const float* gscale, int e0, int E, float hs) {
  if constexpr (FP8) {
    if (e0 + 32 <= E) {  // e0 is a multiple of 32 and gscale 16-byte aligned: eight 16-byte loads
      const float4* g4 = reinterpret_cast<const float4*>(gscale + e0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 g = __ldg(g4 + q);
        r[4 * q + 0] = __float_as_uint(__uint_as_float(r[4 * q + 0]) * g.x * hs);
        r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) * g.y * hs);
        r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) * g.z * hs);
        r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) * g.w * hs);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = min(e0 + j, E - 1);
        r[j] = __float_as_uint(__uint_as_float(r[j]) * __ldg(gscale + e) * hs);
      }
    }
  }
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Shared-memory descriptors of K slice kk (0..3) of a stage.
//  A, K-major SW128: rows of 128 B, 8-row groups 1024 B apart (SBO); the
//    16-element K slice starts 32 B further into each swizzled row.
//  B, MN-major SW128: 64-expert blocks 8 KB apart (LBO), 8-row K groups 1024 B
//    apart (SBO); a 16-row K slice starts 2 groups (2048 B) further.
__device__ __forceinline__ uint64_t a_desc_k_slice(uint32_t a_stage_addr, int kk) {
  return smem_desc_sw128(a_stage_addr + kk * (UMMA_K * 2), 16, 1024);
}
__device__ __forceinline__ uint64_t b_desc_k_slice(uint32_t b_stage_addr, int kk) {
  return smem_desc_sw128(b_stage_addr + kk * (UMMA_K / 8) * 1024, B_BOX_BYTES, 1024);
}

template <bool FP8>
__device__ __forceinline__ uint64_t gate_desc_k_slice(uint32_t b_addr, int kk) {
  if constexpr (FP8)
    return smem_desc_sw128(b_addr + kk * 32, 16, 1024);
  else
    return b_desc_k_slice(b_addr, kk);
}

constexpr int E_GROUP = 512;  // experts per group: the MMA N that fits tensor memory

// The MMA shape of expert group g: n_pad columns in n_chunks chunks.
struct GroupShape {
  int e0;        // first expert of the group
  int n_pad;     // MMA N of the group
  int n_chunks;  // ceil(n_pad / 256)
};

__device__ __forceinline__ GroupShape group_shape(const RowTileParams& p, int g) {
  GroupShape s;
  s.e0 = g * E_GROUP;
  s.n_pad = g == 0 ? min(p.n_pad, E_GROUP) : p.n_pad - E_GROUP;
  s.n_chunks = (s.n_pad + N_CHUNK - 1) / N_CHUNK;
  return s;
}

// Width of MMA chunk c of a group (all but the last are N_CHUNK wide).
__device__ __forceinline__ int chunk_n(const GroupShape& s, int c) {
  return c + 1 < s.n_chunks ? N_CHUNK : s.n_pad - N_CHUNK * (s.n_chunks - 1);
}

// Gate boxes (64 experts each) of chunk c that one CTA stages per K slice.
template <int CG>
__device__ __forceinline__ int chunk_boxes(const GroupShape& s, int c) {
  return (chunk_n(s, c) / CG + B_BOX_N - 1) / B_BOX_N;
}

// The i-th tile of a CTA (or pair) `unit` out of `units`: full tiles round-robin,
// then at most one half tile.  Returns false past the end of its list.
struct TileWork {
  int row0;   // first token row of the tile (pair tile: of the pair)
  bool half;  // 128-token pair tile
  int eg;     // expert group of this work item
  int kb0;    // K slices [kb0, kb1) of this item: all of H unless split
  int kb1;
  int split;  // 0: a whole tile; 1 / 2: the first / second H half of split tile `sidx`
  int sidx;
};

template <int CG, int EG, bool SPLIT>
__device__ __forceinline__ bool tile_work(const RowTileParams& p, int unit, int units, int item, TileWork& w) {
  // every tile is EG (1 or 2) consecutive work items, one per expert group
  const int i = EG == 1 ? item : item >> 1;
  w.eg = EG == 1 ? 0 : item & 1;
  w.kb0 = 0;
  w.kb1 = p.k_blocks;
  w.split = 0;
  w.sidx = 0;
  const int n_full = unit < p.num_tiles ? (p.num_tiles - 1 - unit) / units + 1 : 0;
  if (i < n_full) {
    w.row0 = (unit + i * units) * (BLOCK_M * CG);
    w.half = false;
    return true;
  }
  if (SPLIT && i == n_full && unit < 2 * p.num_split) {
    w.sidx = unit >> 1;
    w.split = 1 + (unit & 1);
    w.row0 = (p.num_tiles + w.sidx) * (BLOCK_M * CG);
    w.half = false;
    w.kb0 = w.split == 1 ? 0 : p.split_kb;
    w.kb1 = w.split == 1 ? p.split_kb : p.k_blocks;
    return true;
  }
  if (CG == 2 && i == n_full && unit < p.num_half) {
    w.row0 = p.num_tiles * (BLOCK_M * CG) + unit * BLOCK_M;
    w.half = true;
    return true;
  }
  return false;
}

// Offer 32 consecutive logits (accumulator columns c0 .. c0+31, expert ids
// col_base + c0 ..) of this thread's row; columns at or beyond ncols (MMA
// padding) are skipped.
// Verification aid: store 32 consecutive logits of one row (experts e0 ..
// e0+31, those below `limit`) into the row-major [T, E] array `logits`.
__device__ __forceinline__ void store_logit_chunk(float* logits, int64_t row, int E, int e0, int limit,
                                                  const uint32_t (&r)[32]) {
  float* dst = logits + row * E + e0;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (e0 + j < limit) dst[j] = __uint_as_float(r[j]);
}

template <int KMAX>
__device__ __forceinline__ void offer_chunk(RowTopK<KMAX>& top, const uint32_t (&r)[32], int c0, int ncols,
                                            int col_base) {
  if (c0 + 32 <= ncols) {
#pragma unroll
    for (int j = 0; j < 32; ++j) top.offer(__uint_as_float(r[j]), col_base + c0 + j);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < ncols) top.offer(__uint_as_float(r[j]), col_base + c0 + j);
  }
}

// Split last round: wait (one thread) until *flag == want, bounded like the
// mbarrier waits; false (abort flag and error bit set) when the limit expires
// or the CTA has already aborted.
__device__ __forceinline__ bool wait_split_flag(const uint32_t* flag, uint32_t want, volatile int* abort,
                                                uint64_t timeout_ns, uint32_t* err_word) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == want) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort = 1;
      atomicOr(err_word, ERR_WAIT_EPILOGUE);
      return false;
    }
    __nanosleep(256);
  }
}

// r[j] <- other[j] + r[j] for the 32 floats of a chunk (the first H half's
// partial, staged in shared memory, plus this CTA's own, in that order).
__device__ __forceinline__ void add_first_half(uint32_t (&r)[32], const float* other) {
  const float4* o = reinterpret_cast<const float4*>(other);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = o[q];
    r[4 * q + 0] = __float_as_uint(v.x + __uint_as_float(r[4 * q + 0]));
    r[4 * q + 1] = __float_as_uint(v.y + __uint_as_float(r[4 * q + 1]));
    r[4 * q + 2] = __float_as_uint(v.z + __uint_as_float(r[4 * q + 2]));
    r[4 * q + 3] = __float_as_uint(v.w + __uint_as_float(r[4 * q + 3]));
  }
}

// EG: expert groups (compile time, so that the single-group kernel carries no
// group bookkeeping: kept at run time it cost ~4% of the 65536-token kernel's
// cycles).
// SPLIT: the workspace entry points' split last round (pairs, one expert group,
// four epilogue warps; RowTileParams::num_split): compiled into instances of
// its own, so the other instances carry none of its code.
template <int KMAX, int CG, bool FP8, int EG, bool SPLIT = false>
__global__ void __launch_bounds__(row_tile_threads(KMAX, EG), 1)
    gating_row_tiles_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_x64,
                            const __grid_constant__ CUtensorMap map_w, const RowTileParams p) {
  static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair");
  constexpr int NUM_EPI_WARPS = epi_warps(KMAX, EG);
  static_assert(!SPLIT || (CG == 2 && EG == 1 && NUM_EPI_WARPS == 4), "split last round: pairs, one group, four warps");
  constexpr bool kPair = CG == 2;
  const bool clock_cta = p.clock != nullptr && blockIdx.x == 0 && threadIdx.x == 0;
  const uint64_t t0_ns = clock_cta ? globaltimer_ns() : 0;
  const uint64_t t0_clk = clock_cta ? sm_clock64() : 0;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align_1024(smem_dyn);
  uint8_t* sA = smem;
  uint8_t* sB = smem + p.stages * KB_PER_STAGE * A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + p.stages * KB_PER_STAGE * p.b_boxes * B_BOX_BYTES);
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  uint64_t* split_bar = reinterpret_cast<uint64_t*>(tmem_holder + 2);  // split second half: the partial's bulk load
  // eight epilogue warps: hand-over of the second column half's lists of a full
  // tile, 128 rows of KMAX values, then of KMAX ids (the host adds its bytes to
  // the launch's shared memory)
  float* hand_v = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + EPI_BARRIER_RESERVE);
  int32_t* hand_i = reinterpret_cast<int32_t*>(hand_v + BLOCK_M * KMAX);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;  // 0 = the pair's MMA leader
  const bool leader = rank == 0;
  const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], NUM_EPI_WARPS * CG);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain, 1);
    mbar_init(split_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_x);
    if (kPair && p.num_half > 0) tma_prefetch_desc(&map_x64);
    tma_prefetch_desc(&map_w);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(tmem_holder, p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  if constexpr (kPair) {
    // the peer's loads and arrivals target the leader's barriers: both initialised first
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      // The launch may overlap the previous kernel's tail (programmatic dependent
      // launch): every global read and write of this kernel follows this wait,
      // the later ones through the ring's and accumulator's barriers.
      griddep_wait();
      const uint64_t pol_x = l2_policy_evict_first();  // hidden: streamed once
      const uint64_t pol_w = l2_policy_evict_last();   // gate: re-read by every tile
      // gate box j of a K slice starts at column j * 64 + (j < bpc0 ? col_a : col_b): this
      // CTA's share of chunk 0 (bpc0 boxes), then of chunk 1 (starting at expert 256)
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      TileWork w;
      for (int item = 0; ok && tile_work<CG, EG, SPLIT>(p, unit, units, item, w); ++item) {
        const int cta_rows = w.half ? BLOCK_M / 2 : BLOCK_M;  // hidden rows this CTA stages
        const int row0 = w.row0 + static_cast<int>(rank) * cta_rows;
        // this work item's gate boxes: box j of a K slice starts at expert
        // j * 64 + (j < bpc0 ? col_a : col_b), this CTA's share of chunk 0 (bpc0
        // boxes), then of chunk 1 (from the group's expert 256)
        const GroupShape gs = group_shape(p, w.eg);
        const int bpc0 = chunk_boxes<CG>(gs, 0);
        const int boxes = bpc0 + (gs.n_chunks > 1 ? chunk_boxes<CG>(gs, 1) : 0);
        const int col_a = gs.e0 + static_cast<int>(rank) * (chunk_n(gs, 0) / CG);
        const int col_b =
            gs.n_chunks > 1 ? gs.e0 + N_CHUNK + static_cast<int>(rank) * (chunk_n(gs, 1) / CG) - bpc0 * B_BOX_N : 0;
        const uint32_t stage_tx = KB_PER_STAGE * CG * (cta_rows * BLOCK_K * 2 + boxes * B_BOX_BYTES);
        const CUtensorMap* map_a = w.half ? &map_x64 : &map_x;
        // K slices past H (when k_blocks is odd) are out of bounds: TMA fills zeros
        for (int kb = w.kb0; kb < w.kb1; kb += KB_PER_STAGE) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns, ERR_WAIT_PRODUCER, p.err_word)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
#pragma unroll
          for (int sub = 0; sub < KB_PER_STAGE; ++sub) {
            const int slot = stage * KB_PER_STAGE + sub;
            const int k0 = (kb + sub) * slice_k<FP8>();
            // gate box coordinates: bf16 [H, E] map (x = expert, y = K), FP8 [E, H] map (x = K, y = expert)
            if constexpr (kPair) {
              const uint32_t bar = map_shared_rank(smem_u32(&full[stage]), 0);
              tma_load_2d_pair(sA + slot * A_STAGE_BYTES, map_a, bar, k0, row0, pol_x);
              for (int j = 0; j < boxes; ++j) {
                const int col = j * B_BOX_N + (j < bpc0 ? col_a : col_b);
                tma_load_2d_pair(sB + (slot * p.b_boxes + j) * B_BOX_BYTES, &map_w, bar, FP8 ? k0 : col,
                                 FP8 ? col : k0, pol_w);
              }
            } else {
              tma_load_2d(sA + slot * A_STAGE_BYTES, &map_x, &full[stage], k0, row0, pol_x);
              for (int j = 0; j < boxes; ++j) {
                const int col = j * B_BOX_N + (j < bpc0 ? col_a : col_b);
                tma_load_2d(sB + (slot * p.b_boxes + j) * B_BOX_BYTES, &map_w, &full[stage], FP8 ? k0 : col,
                            FP8 ? col : k0, pol_w);
              }
            }
          }
          ++issued;
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Every load issued lands before the CTA may exit.  The leader's full
      // barriers count both CTAs' bytes; the peer's loads are covered by the
      // leader's drain and the closing cluster barrier.
      if (leader) {
        const int pending = issued < p.stages ? issued : p.stages;
        for (int n = 0; n < pending; ++n) {
          if (stage == 0) {
            stage = p.stages - 1;
            phase ^= 1;
          } else {
            --stage;
          }
          mbar_wait(&full[stage], phase, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer ----------------
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int local = 0;
      TileWork w;
      for (; ok && tile_work<CG, EG, SPLIT>(p, unit, units, local, w); ++local) {
        const uint32_t buf = static_cast<uint32_t>(local % p.acc_bufs);
        const uint32_t acc_phase = static_cast<uint32_t>(local / p.acc_bufs) & 1;
        // this work item's chunks: instruction descriptors (pairs: M = 128 for a
        // half tile) and the offset of chunk 1's gate boxes within a K slice
        const GroupShape gs = group_shape(p, w.eg);
        const bool two_chunks = gs.n_chunks > 1;
        const uint32_t m = w.half ? BLOCK_M : BLOCK_M * CG;
        const uint32_t id0 = mma_idesc<FP8>(m, chunk_n(gs, 0));
        const uint32_t id1 = mma_idesc<FP8>(m, two_chunks ? chunk_n(gs, 1) : N_CHUNK);
        const uint32_t b_off1 = static_cast<uint32_t>(chunk_boxes<CG>(gs, 0) * B_BOX_BYTES);
        if (!mbar_wait(&acc_empty[buf], acc_phase ^ 1, abort_flag, p.timeout_ns, ERR_WAIT_MMA, p.err_word)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + buf * p.acc_stride;
        for (int kb = w.kb0; kb < w.kb1; kb += KB_PER_STAGE) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.timeout_ns, ERR_WAIT_MMA, p.err_word)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
#pragma unroll
          for (int sub = 0; sub < KB_PER_STAGE; ++sub) {
            const int slot = stage * KB_PER_STAGE + sub;
            const uint32_t a_addr = smem_u32(sA + slot * A_STAGE_BYTES);
            const uint32_t b_addr = smem_u32(sB + slot * p.b_boxes * B_BOX_BYTES);
            // the chunk count is loop-invariant: one branch per slice, none per MMA
            // (extra work between MMAs measurably slows the issue loop)
            if (two_chunks) {
#pragma unroll
              for (int kk = 0; kk < BLOCK_K / UMMA_K; ++kk) {
                const uint32_t accumulate = ((kb - w.kb0 + sub) | kk) != 0;
                const uint64_t a_desc = a_desc_k_slice(a_addr, kk);
                umma<FP8, kPair>(d_tmem, a_desc, gate_desc_k_slice<FP8>(b_addr, kk), id0, accumulate);
                umma<FP8, kPair>(d_tmem + N_CHUNK, a_desc, gate_desc_k_slice<FP8>(b_addr + b_off1, kk), id1,
                                 accumulate);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < BLOCK_K / UMMA_K; ++kk) {
                const uint32_t accumulate = ((kb - w.kb0 + sub) | kk) != 0;
                umma<FP8, kPair>(d_tmem, a_desc_k_slice(a_addr, kk), gate_desc_k_slice<FP8>(b_addr, kk), id0,
                                 accumulate);
              }
            }
          }
          // frees the stage (in both CTAs of a pair) once these MMAs have read it
          if constexpr (kPair)
            umma_commit_pair_multicast(&empty[stage], 0x3);
          else
            umma_commit(&empty[stage]);
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) {
          if constexpr (kPair)
            umma_commit_pair_multicast(&acc_full[buf], 0x3);
          else
            umma_commit(&acc_full[buf]);
        }
      }
      // Every MMA issued completes before tensor memory is freed.
      if constexpr (kPair)
        umma_commit_pair(drain);
      else
        umma_commit(drain);
      mbar_wait(drain, 0, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;       // TMEM lanes this warp may access
    const int hc = (warp - 2) >> 2;  // column half of this warp (0: warps 2..5, 1: warps 6..9)
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    int local = 0;
    TileWork w;
    RowTopK<KMAX> top;
    for (; tile_work<CG, EG, SPLIT>(p, unit, units, local, w); ++local) {
      const uint32_t buf = static_cast<uint32_t>(local % p.acc_bufs);
      const uint32_t acc_phase = static_cast<uint32_t>(local / p.acc_bufs) & 1;
      const bool ok = mbar_wait(&acc_full[buf], acc_phase, abort_flag, p.timeout_ns, ERR_WAIT_EPILOGUE, p.err_word);
      // The four epilogue warps take one decision: a warp that went on alone
      // after the others gave up would wait for them forever at the half
      // tile's list exchange below.
      if (!named_barrier_and(2, NUM_EPI_WARPS * 32, ok)) break;
      tc_fence_after_sync();

      // split last round (pairs, one expert group, four epilogue warps)
      const float* first_half = nullptr;  // second H half: the stored first-half partial of this thread's row
      if constexpr (SPLIT) {
        if (w.split == 1) {
          // First H half: this CTA's 128 accumulator rows, columns [0, part_cols)
          // (column c = expert c), to the workspace.  As in a half tile, this is
          // the CTA's last item and its ring is idle: each warp moves its 32 rows
          // in 32-column chunks through a padded tile there, so that every store
          // instruction writes four whole 128-byte rows of a chunk.
          const uint32_t acc_addr = lane_base + buf * p.acc_stride;
          float* xpose = reinterpret_cast<float*>(sA) + quad * (32 * XPOSE_STRIDE);
          const int row_in_tile = rank * BLOCK_M + quad * 32;  // this warp's first row of the 256
          const int64_t row_base = static_cast<int64_t>(w.row0) + row_in_tile;
          float* dst = p.split_part + (static_cast<int64_t>(w.sidx) * (2 * BLOCK_M) + row_in_tile) * p.part_stride;
          const int qc = 4 * (lane & 7);
          if (TK_CHECK(NUM_EPI_WARPS * 32 * XPOSE_STRIDE * 4 <= p.stages * KB_PER_STAGE * A_STAGE_BYTES, p.err_word)) {
            for (int c0 = 0; c0 < p.part_cols; c0 += 32) {
              uint32_t r[32];
              if (!TK_CHECK(((acc_addr - tmem_base) & 0xFFFFu) + c0 + 32u <= p.tmem_cols, p.err_word)) break;
              tmem_ld_32(acc_addr + c0, r);
              tmem_ld_wait();
              float* mine = xpose + lane * XPOSE_STRIDE;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(mine + j) = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                                   __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
              __syncwarp();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int rr = 4 * i + (lane >> 3);
                const float4 v = *reinterpret_cast<const float4*>(xpose + rr * XPOSE_STRIDE + qc);
                if (row_base + rr < p.T)
                  *reinterpret_cast<float4*>(dst + static_cast<int64_t>(rr) * p.part_stride + c0 + qc) = v;
              }
              __syncwarp();
            }
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if (!leader)
              mbar_arrive_remote(map_shared_rank(smem_u32(&acc_empty[buf]), 0));
            else
              mbar_arrive(&acc_empty[buf]);
          }
          // every warp's rows are stored: publish them to the second half's pair
          named_barrier_sync(4, NUM_EPI_WARPS * 32);
          if (warp == 2 && lane == 0) {
            __threadfence();
            atomicExch(p.split_flags + 2 * w.sidx + rank, p.split_token);
          }
          continue;
        }
        if (w.split == 2) {
          // Second H half: one thread waits (bounded) until the first half's pair
          // has stored the same rows, then brings this CTA's 128 of them --
          // contiguous in the workspace -- into the idle ring (this is the CTA's
          // last item) with one bulk copy; the warps agree on the outcome, and
          // each thread then reads its row there.
          const uint32_t rows_bytes = static_cast<uint32_t>(BLOCK_M * p.part_stride * 4);
          bool got = true;
          bool issued = false;
          if (warp == 2 && lane == 0) {
            got = wait_split_flag(p.split_flags + 2 * w.sidx + rank, p.split_token, abort_flag, p.timeout_ns,
                                  p.err_word);
            // the rows land in the idle ring (its hidden-row and gate parts together)
            if (got && TK_CHECK(rows_bytes <= static_cast<uint32_t>(p.stages * KB_PER_STAGE *
                                                                    (A_STAGE_BYTES + p.b_boxes * B_BOX_BYTES)),
                                p.err_word)) {
              fence_proxy_async_global();  // the flag was acquired by ordinary loads; the copy reads asynchronously
              mbar_arrive_expect_tx(split_bar, rows_bytes);
              bulk_load_g2s(sA,
                            p.split_part + (static_cast<int64_t>(w.sidx) * (2 * BLOCK_M) + rank * BLOCK_M) * p.part_stride,
                            rows_bytes, split_bar);
              issued = true;
            } else {
              got = false;
            }
          }
          got = named_barrier_and(4, NUM_EPI_WARPS * 32, got);
          if (got) {
            got = mbar_wait(split_bar, 0, abort_flag, p.timeout_ns, ERR_WAIT_EPILOGUE, p.err_word);
            got = named_barrier_and(4, NUM_EPI_WARPS * 32, got);
            // a copy still in flight after an expired wait lands before the CTA may exit
            if (!got && issued) mbar_wait(split_bar, 0, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
          }
          if (got) first_half = reinterpret_cast<const float*>(sA) + (quad * 32 + lane) * p.part_stride;
        }
      }

      // full tile: one row per thread, TMEM column c = expert e0 + c of the group;
      // half tile: per chunk c, lanes 0..63 hold experts e0 + [256c, 256c + N_c/2)
      // and lanes 64..127 experts e0 + [256c + N_c/2, 256c + N_c) of 64 rows, in
      // columns from 256c
      const bool upper = w.half && quad >= 2;
      if (w.eg == 0) top.reset();  // the lists run over every expert group of the tile
      const uint32_t acc_addr = lane_base + buf * p.acc_stride;
      const GroupShape gs = group_shape(p, w.eg);
      const int64_t my_row = w.half ? static_cast<int64_t>(w.row0) + rank * (BLOCK_M / 2) + (quad & 1) * 32 + lane
                                    : static_cast<int64_t>(w.row0) + rank * BLOCK_M + quad * 32 + lane;
      float hs = 1.0f;  // FP8: this row's token scale
      if constexpr (FP8) hs = my_row < p.T ? __ldg(p.hscale + my_row) : 0.0f;
      const bool dump = p.logits != nullptr && my_row < p.T;
      // full tiles: one pass over the group's columns; half tiles: one per chunk
      const int passes = w.half ? gs.n_chunks : 1;
      for (int c = 0; c < passes; ++c) {
        int col_base = gs.e0, ncols = min(gs.n_pad, p.E - gs.e0);
        uint32_t chunk_addr = acc_addr;
        if (w.half) {
          col_base = gs.e0 + c * N_CHUNK + (upper ? chunk_n(gs, c) / 2 : 0);
          ncols = min(chunk_n(gs, c) / 2, p.E - col_base);
          chunk_addr += static_cast<uint32_t>(c * N_CHUNK);
        }
        // this warp's half of the pass's columns: [0, mid) or [mid, ncols), mid a
        // multiple of 32 (one tensor-memory load)
        const int mid = NUM_EPI_WARPS == 4 ? ncols : min(ncols, (ncols + 63) / 64 * 32);
        const int lo = hc == 0 ? 0 : mid;
        const int hi = hc == 0 ? mid : ncols;
        // 64 columns per round trip: two loads, one wait
        for (int c0 = lo; c0 < hi; c0 += 64) {
          uint32_t r0[32], r1[32];
          const bool second = c0 + 32 < hi;  // warp-uniform
          // the columns read stay inside this CTA's tensor-memory allocation
          if (!TK_CHECK(((chunk_addr - tmem_base) & 0xFFFFu) + c0 + (second ? 64u : 32u) <= p.tmem_cols, p.err_word))
            break;
          tmem_ld_32(chunk_addr + c0, r0);
          if (second) tmem_ld_32(chunk_addr + c0 + 32, r1);
          tmem_ld_wait();
          if constexpr (SPLIT) {
            if (first_half != nullptr) {  // split second half: add the first half's partial (full tiles: c = column)
              add_first_half(r0, first_half + c0);
              if (second) add_first_half(r1, first_half + c0 + 32);
            }
          }
          scale_chunk<FP8>(r0, p.gscale, col_base + c0, p.E, hs);
          if (dump) store_logit_chunk(p.logits, my_row, p.E, col_base + c0, col_base + hi, r0);
          offer_chunk(top, r0, c0, hi, col_base);
          if (second) {
            scale_chunk<FP8>(r1, p.gscale, col_base + c0 + 32, p.E, hs);
            if (dump) store_logit_chunk(p.logits, my_row, p.E, col_base + c0 + 32, col_base + hi, r1);
            offer_chunk(top, r1, c0 + 32, hi, col_base);
          }
        }
      }
      // the accumulator buffer may be overwritten once every epilogue warp of
      // the pair has read it
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (kPair && !leader)
          mbar_arrive_remote(map_shared_rank(smem_u32(&acc_empty[buf]), 0));
        else
          mbar_arrive(&acc_empty[buf]);
      }

      if constexpr (SPLIT) {
        if (w.split == 2) {
          // every warp has read the first half's partial: clear the flag for the next call
          named_barrier_sync(4, NUM_EPI_WARPS * 32);
          if (warp == 2 && lane == 0 && first_half != nullptr) atomicExch(p.split_flags + 2 * w.sidx + rank, 0u);
        }
      }
      if (w.eg + 1 < EG) continue;  // the tile's next expert group follows
      if (!w.half) {
        // the second half's list of each row goes to the first half's thread of
        // that row (the next tile's lists are written only after every epilogue
        // warp has passed the next tile's agreement barrier, i.e. after these reads)
        if constexpr (NUM_EPI_WARPS == 8) {
          float* xv = hand_v + (quad * 32 + lane) * KMAX;
          int32_t* xi = hand_i + (quad * 32 + lane) * KMAX;
          if (hc == 1) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
              xv[j] = top.v[j];
              xi[j] = top.i[j];
            }
          }
          named_barrier_sync(3, NUM_EPI_WARPS * 32);
          if (hc == 0) {
            float bv[KMAX];
            int32_t bi[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
              bv[j] = xv[j];
              bi[j] = xi[j];
            }
            merge_sorted(top, bv, bi);
          }
        }
        if (hc == 0) {
          const int64_t row = static_cast<int64_t>(w.row0) + rank * BLOCK_M + quad * 32 + lane;
          if (row < p.T) {
            top.softmax_store(p.k, p.scores + row * p.k, p.ids + row * p.k);
            if (p.route.table != nullptr) route_count_row(p.route, top, p.k, row, p.E);
          }
        }
      } else {
        // A half tile is a CTA's last tile (and this its last expert group), so
        // its ring is idle: each of a row's four lists (lane half x column half)
        // but the lower lanes' first half goes through it to that thread.
        const int m = (quad & 1) * 32 + lane;  // row within this CTA's 64
        const int slot = (upper ? 2 : 0) + hc;  // this thread's list of row m
        // the hand-over area (64 rows x 4 lists of KMAX floats, then of KMAX ids) lies inside the idle ring
        if (!TK_CHECK(4 * (BLOCK_M / 2) * KMAX * 8 <= p.stages * KB_PER_STAGE * A_STAGE_BYTES, p.err_word)) break;
        float* xv = reinterpret_cast<float*>(sA) + m * 4 * KMAX;
        int32_t* xi = reinterpret_cast<int32_t*>(sA + 4 * (BLOCK_M / 2) * KMAX * 4) + m * 4 * KMAX;
        if (slot != 0) {
#pragma unroll
          for (int j = 0; j < KMAX; ++j) {
            xv[slot * KMAX + j] = top.v[j];
            xi[slot * KMAX + j] = top.i[j];
          }
        }
        named_barrier_sync(1, NUM_EPI_WARPS * 32);
        if (slot == 0) {
          for (int o = 1; o < 4; ++o) {
            if (NUM_EPI_WARPS == 4 && (o & 1)) continue;  // four warps: no second column half
            float bv[KMAX];
            int32_t bi[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
              bv[j] = xv[o * KMAX + j];
              bi[j] = xi[o * KMAX + j];
            }
            merge_sorted(top, bv, bi);
          }
          const int64_t row = static_cast<int64_t>(w.row0) + rank * (BLOCK_M / 2) + m;
          if (row < p.T) {
            top.softmax_store(p.k, p.scores + row * p.k, p.ids + row * p.k);
            if (p.route.table != nullptr) route_count_row(p.route, top, p.k, row, p.E);
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  if constexpr (kPair) {
    settle_after_abort(abort_flag);
    // neither CTA frees its shared or tensor memory while the pair still uses it
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else
      tmem_dealloc(tmem_base, p.tmem_cols);
  }
  if (clock_cta) record_launch_clock(p.clock, t0_ns, t0_clk);
}

}  // namespace tkg
