// Fused gating for few tokens: a cluster of C CTAs shares one 128-token tile
// and splits the hidden dimension H between its CTAs.
//
// With T <= a few thousand tokens there are too few 128-token tiles to occupy
// the GPU (T = 1..128 is a single tile), while every tile still streams the whole
// gate matrix (H x E).  Here CTA r of the cluster accumulates the logits over
// its own slice of H on the tensor cores:
//
//   1. mainloop (as in the row-tile kernel, one tile, k-blocks [kb0, kb1)):
//      partial_r[128, E] in tensor memory;
//   2. once its own ring is idle, every CTA copies its partial rows from tensor
//      memory into its own shared memory (local stores only);
//   3. cluster barrier: every CTA's partial rows are visible to the cluster;
//   4. CTA r owns the tile rows t with t % C == r.  Each owned row is split
//      into G column segments, one thread each: the thread reads the C
//      partials of its segment -- its own from local shared memory, the others
//      straight from the other CTAs' shared memory (distributed shared memory
//      loads: the owner pulls) -- adds them in rank order 0..C-1 (so a logit
//      does not depend on which CTA owns its row), keeps a top-k of the
//      segment, and the G lists are merged with warp shuffles; then softmax
//      and store;
//   5. cluster barrier: no CTA reuses or releases its shared memory while an
//      owner may still read it.
//
// More than 256 experts (up to 512): one MMA per chunk of at most 256 experts
// and K step (chunk c in tensor-memory columns from 256c), and steps 2..4 run
// once per 256-expert column range (with a cluster barrier between passes):
// each pass stages and reduces its columns and the owners keep their running
// top-k lists across passes.  More than 512
// (up to 1024): steps 1..5 run once per group of 512 experts, the ring position
// carried over; the owners' lists run over both groups.
//
// FP8 = true: E4M3 inputs as in the row-tile kernel (kind::f8f6f4, K-major
// expert-major gate, 128 K values per slice); owners scale the summed logits
// by the token's and the expert's scale before selecting.
//
// Nothing but scores and ids is written to global memory (and, when the
// verification array `logits` is given, every summed logit of the tile).
#pragma once

#include <cuda.h>
#include <cstdint>

#include "gating_row_tiles.cuh"
#include "sm100_ptx.cuh"
#include "topk_epilogue.cuh"
#include "route_counts.cuh"
#include "topk_merge.cuh"

namespace tkg {

// Warps: 0 producer, 1 MMA, 2..5 stage partial rows (TMEM lane quadrants), 6..7
// join the reduction; all 8 reduce.
constexpr int SPLIT_THREADS = 256;
constexpr int SPLIT_WARPS = SPLIT_THREADS / 32;
constexpr int PUSH_WARPS = 4;

struct SplitHParams {
  int32_t T, H, E, k;
  int32_t n_pad;        // total MMA N (E rounded up to 16, <= 1024)
  int32_t e_groups;     // expert groups of at most 512 (1 or 2), computed one after the other
  int32_t kps;          // K slices per ring stage (2, or 1 when n_pad > 256)
  int32_t num_tiles;    // 128-token tiles
  int32_t k_blocks;     // ceil(H / 64)
  int32_t stages;
  int32_t b_boxes;      // gate boxes per K slice in the ring (group 0's count, the largest)
  int32_t row_stride;   // floats per staged partial row (round_up(min(E, 256), 32) + 4)
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
};

template <int KMAX, int C, bool FP8>
__global__ void __launch_bounds__(SPLIT_THREADS, 1)
    gating_split_h_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                          const SplitHParams p) {
  const bool clock_cta = p.clock != nullptr && blockIdx.x == 0 && threadIdx.x == 0;
  const uint64_t t0_ns = clock_cta ? globaltimer_ns() : 0;
  const uint64_t t0_clk = clock_cta ? sm_clock64() : 0;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align_1024(smem_dyn);
  uint8_t* sA = smem;
  uint8_t* sB = smem + p.stages * p.kps * A_STAGE_BYTES;
  float* staging = reinterpret_cast<float*>(smem);  // reuses the ring once every CTA's MMAs are done
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + p.stages * p.kps * p.b_boxes * B_BOX_BYTES);  // after the ring
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t r = cluster_ctarank();
  const int tile = static_cast<int>(blockIdx.x / C);
  // balanced split of the k-blocks; non-empty for every CTA since C <= k_blocks
  const int kb0 = static_cast<int>((static_cast<int64_t>(r) * p.k_blocks) / C);
  const int kb1 = static_cast<int>((static_cast<int64_t>(r + 1) * p.k_blocks) / C);
  const int valid_rows = min(BLOCK_M, p.T - tile * BLOCK_M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, p.tmem_cols);
    tmem_relinquish();
  }
  // The launch may overlap the previous kernel's tail (programmatic dependent
  // launch); the set-up above touches no global memory, everything below may.
  griddep_wait();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  // Owned rows: n_own <= 64 (C >= 2), and group * n_own <= SPLIT_THREADS, so one
  // pass over the owned rows covers them all.  The owners' lists run over every
  // expert group.
  const int n_own = valid_rows > static_cast<int>(r) ? (valid_rows - static_cast<int>(r) + C - 1) / C : 0;
  int group = 32;  // threads per owned row: a power of two
  while (group > 1 && (n_own * group > SPLIT_THREADS || group * 8 > min(p.E, N_CHUNK))) group >>= 1;
  const int slot = static_cast<int>(threadIdx.x) / group;
  const int seg = threadIdx.x % group;
  const bool active = slot < n_own;
  RowTopK<KMAX> top;
  top.reset();

  // ring position of the producer (warp 0) and of the MMA issuer (warp 1),
  // carried from one expert group to the next
  uint32_t ring_stage = 0, ring_phase = 0;

  for (int eg = 0; eg < p.e_groups; ++eg) {
    // expert group eg: experts [512 eg, 512 eg + np), np = its MMA N, in chunks of 256
    const int e0 = eg * E_GROUP;
    const int np = eg == 0 ? min(p.n_pad, E_GROUP) : p.n_pad - E_GROUP;
    const int n_chunks = (np + N_CHUNK - 1) / N_CHUNK;
    const int boxes = (np + B_BOX_N - 1) / B_BOX_N;
    const uint32_t parity = static_cast<uint32_t>(eg) & 1;

    if (warp == 0) {
      if (lane == 0) {
        // ---------------- TMA producer: this CTA's H slice of one tile ----------------
        const uint64_t pol_x = l2_policy_evict_first();
        const uint64_t pol_w = l2_policy_evict_last();
        const uint32_t slice_tx = A_STAGE_BYTES + boxes * B_BOX_BYTES;
        int issued = 0;
        // after an abort no later expert group is loaded
        for (int kb = *abort_flag ? kb1 : kb0; kb < kb1; kb += p.kps) {
          // a stage holds up to kps slices, never past this CTA's H slice
          const int n_sub = min(p.kps, kb1 - kb);
          if (!mbar_wait(&empty[ring_stage], ring_phase ^ 1, abort_flag, p.timeout_ns, ERR_WAIT_PRODUCER,
                         p.err_word))
            break;
          mbar_arrive_expect_tx(&full[ring_stage], n_sub * slice_tx);
          for (int sub = 0; sub < n_sub; ++sub) {
            const int slot_i = ring_stage * p.kps + sub;
            const int k0 = (kb + sub) * slice_k<FP8>();
            tma_load_2d(sA + slot_i * A_STAGE_BYTES, &map_x, &full[ring_stage], k0, tile * BLOCK_M, pol_x);
            // gate box coordinates: bf16 [H, E] map (x = expert, y = K), FP8 [E, H] map (x = K, y = expert)
            for (int j = 0; j < boxes; ++j) {
              const int col = e0 + j * B_BOX_N;
              tma_load_2d(sB + (slot_i * p.b_boxes + j) * B_BOX_BYTES, &map_w, &full[ring_stage], FP8 ? k0 : col,
                          FP8 ? col : k0, pol_w);
            }
          }
          ++issued;
          if (++ring_stage == static_cast<uint32_t>(p.stages)) {
            ring_stage = 0;
            ring_phase ^= 1;
          }
        }
        // every load of this group lands before the ring is reused for the exchange
        uint32_t ds = ring_stage, dph = ring_phase;
        const int pending = issued < p.stages ? issued : p.stages;
        for (int n = 0; n < pending; ++n) {
          if (ds == 0) {
            ds = p.stages - 1;
            dph ^= 1;
          } else {
            --ds;
          }
          mbar_wait(&full[ds], dph, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------- MMA issuer ----------------
        // chunk c of the group: N = min(256, np - 256c); its gate boxes start at box 4c
        const uint32_t idesc0 = mma_idesc<FP8>(BLOCK_M, min(np, N_CHUNK));
        const uint32_t idesc1 = mma_idesc<FP8>(BLOCK_M, np > N_CHUNK ? np - N_CHUNK : N_CHUNK);
        const bool two_chunks = n_chunks > 1;
        // after an abort no later expert group is computed
        bool ok = *abort_flag == 0;
        for (int kb = kb0; ok && kb < kb1; kb += p.kps) {
          const int n_sub = min(p.kps, kb1 - kb);
          if (!mbar_wait(&full[ring_stage], ring_phase, abort_flag, p.timeout_ns, ERR_WAIT_MMA, p.err_word)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          for (int sub = 0; sub < n_sub; ++sub) {
            const int slot_i = ring_stage * p.kps + sub;
            const uint32_t a_addr = smem_u32(sA + slot_i * A_STAGE_BYTES);
            const uint32_t b_addr = smem_u32(sB + slot_i * p.b_boxes * B_BOX_BYTES);
            if (two_chunks) {  // loop-invariant: no branch between the MMAs of a slice
#pragma unroll
              for (int kk = 0; kk < BLOCK_K / UMMA_K; ++kk) {
                const uint32_t accumulate = (kb + sub != kb0) | kk;
                const uint64_t a_desc = a_desc_k_slice(a_addr, kk);
                umma<FP8, false>(tmem_base, a_desc, gate_desc_k_slice<FP8>(b_addr, kk), idesc0, accumulate);
                umma<FP8, false>(tmem_base + N_CHUNK, a_desc,
                                 gate_desc_k_slice<FP8>(b_addr + (N_CHUNK / B_BOX_N) * B_BOX_BYTES, kk), idesc1,
                                 accumulate);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < BLOCK_K / UMMA_K; ++kk)
                umma<FP8, false>(tmem_base, a_desc_k_slice(a_addr, kk), gate_desc_k_slice<FP8>(b_addr, kk), idesc0,
                                 (kb + sub != kb0) | kk);
            }
          }
          umma_commit(&empty[ring_stage]);
          if (++ring_stage == static_cast<uint32_t>(p.stages)) {
            ring_stage = 0;
            ring_phase ^= 1;
          }
        }
        // committed for every group, finished or not, so that the barrier's
        // phases follow the groups; the push warps check the abort flag
        umma_commit(acc_full);
        umma_commit(drain);
        mbar_wait(drain, parity, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
      }
      __syncwarp();
    }

    // The staging warps wait for this CTA's accumulator.
    const bool push_warp = warp >= 2 && warp < 2 + PUSH_WARPS;
    bool acc_ok = true;
    if (push_warp) {
      acc_ok = mbar_wait(acc_full, parity, abort_flag, p.timeout_ns, ERR_WAIT_EPILOGUE, p.err_word);
      acc_ok = __all_sync(0xffffffffu, acc_ok && *abort_flag == 0);
    }

    // This CTA's ring is idle once its producer has drained its loads and its
    // MMAs are done (the push warps waited for acc_full): the partial rows may
    // overwrite it.
    __syncthreads();

    for (int pass = 0; pass < n_chunks; ++pass) {
      const int col0 = pass * N_CHUNK;                        // first TMEM column of this pass
      const int pass_cols = min(N_CHUNK, p.E - (e0 + col0));  // experts e0 + col0 .. of this pass
      // the previous pass's partials have been pulled by every owner
      if (pass > 0) {
        cluster_arrive_release();
        cluster_wait_acquire();
      }

      // ---------------- partial rows into this CTA's own shared memory ----------------
      // Thread = tile row (tensor-memory lane), 32 columns per load; each thread
      // stores its row's 128 contiguous bytes (rows 260 floats apart: the eight
      // lanes of a quarter warp hit 32 distinct banks).
      if (push_warp) {
        const int quad = warp & 3;
        if (acc_ok && quad * 32 < valid_rows) {
          const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(col0);
          const int t = quad * 32 + lane;  // tile-local row of this thread
          float* row = staging + static_cast<size_t>(t) * p.row_stride;
          [[maybe_unused]] const int ring_bytes = p.stages * p.kps * (A_STAGE_BYTES + p.b_boxes * B_BOX_BYTES);
          // 64 columns per tensor-memory round trip
          for (int c0 = 0; c0 < pass_cols; c0 += 64) {
            uint32_t v[2][32];
            const bool second = c0 + 32 < pass_cols;  // warp-uniform
            // tensor-memory columns inside the allocation; staged row inside the idle ring
            if (!TK_CHECK(col0 + c0 + (second ? 64 : 32) <= static_cast<int>(p.tmem_cols) &&
                              (BLOCK_M - 1) * p.row_stride * 4 + (c0 + (second ? 64 : 32)) * 4 <= ring_bytes &&
                              c0 + (second ? 64 : 32) <= p.row_stride,
                          p.err_word))
              break;
            tmem_ld_32(lane_base + c0, v[0]);
            if (second) tmem_ld_32(lane_base + c0 + 32, v[1]);
            tmem_ld_wait();
            if (t < valid_rows) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                if (h == 1 && !second) break;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                  *reinterpret_cast<float4*>(row + c0 + 32 * h + j) =
                      make_float4(__uint_as_float(v[h][j]), __uint_as_float(v[h][j + 1]),
                                  __uint_as_float(v[h][j + 2]), __uint_as_float(v[h][j + 3]));
              }
            }
          }
        }
      }
      tc_fence_before_sync();
      cluster_arrive_release();  // every CTA's partial rows are visible to the cluster past this point
      cluster_wait_acquire();
      if (warp == 1 && eg + 1 == p.e_groups && pass + 1 == n_chunks) {  // all tensor-memory reads are done
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
      }

      // ---------------- owners pull their rows' partials and reduce ----------------
      // Owner r's row t (t % C == r) sums partial_q[t] over q = 0 .. C-1 in rank
      // order (so a logit does not depend on which CTA owns its row), reading the
      // other CTAs' shared memory directly (distributed shared memory loads).
      if (active) {
        const int t_own = static_cast<int>(r) + C * slot;
        float hs = 1.0f;  // FP8: the row's token scale
        if constexpr (FP8) hs = __ldg(p.hscale + static_cast<int64_t>(tile) * BLOCK_M + t_own);
        const float* mine = staging + static_cast<size_t>(t_own) * p.row_stride;
        const uint32_t mine_addr = smem_u32(mine);
        uint32_t peer[C];
#pragma unroll
        for (int q = 0; q < C; ++q) peer[q] = map_shared_rank(mine_addr, static_cast<uint32_t>(q));
        const int ebase = e0 + col0;
        // segment `seg` takes every group-th float4 of the row: consecutive lanes
        // read consecutive 16-byte words, and each thread still offers its
        // columns in increasing order
        auto column_quad = [&](int c) {
          float4 v[C];
#pragma unroll
          for (int q = 0; q < C; ++q)
            v[q] = q == static_cast<int>(r) ? *reinterpret_cast<const float4*>(mine + c)
                                              : ld_shared_cluster_f4(peer[q] + static_cast<uint32_t>(c) * 4u);
          float4 acc = v[0];
#pragma unroll
          for (int q = 1; q < C; ++q) {  // rank order: the same sum whichever CTA owns the row
            acc.x += v[q].x;
            acc.y += v[q].y;
            acc.z += v[q].z;
            acc.w += v[q].w;
          }
          if constexpr (FP8) {  // expert scales of columns past E are never offered
            const int e = ebase + c;
            acc.x = acc.x * __ldg(p.gscale + min(e, p.E - 1)) * hs;
            acc.y = acc.y * __ldg(p.gscale + min(e + 1, p.E - 1)) * hs;
            acc.z = acc.z * __ldg(p.gscale + min(e + 2, p.E - 1)) * hs;
            acc.w = acc.w * __ldg(p.gscale + min(e + 3, p.E - 1)) * hs;
          }
          return acc;
        };
        float* dump = p.logits == nullptr ? nullptr
                                          : p.logits + (static_cast<int64_t>(tile) * BLOCK_M + t_own) * p.E + ebase;
        for (int c = 4 * seg; c < pass_cols; c += 4 * group) {
          // the pulled columns lie inside the staged row of every CTA
          if (!TK_CHECK(c + 4 <= p.row_stride && t_own < BLOCK_M, p.err_word)) break;
          const float4 acc = column_quad(c);
          if (dump != nullptr) {
            dump[c] = acc.x;
            if (c + 1 < pass_cols) dump[c + 1] = acc.y;
            if (c + 2 < pass_cols) dump[c + 2] = acc.z;
            if (c + 3 < pass_cols) dump[c + 3] = acc.w;
          }
          top.offer(acc.x, ebase + c);
          if (c + 1 < pass_cols) top.offer(acc.y, ebase + c + 1);
          if (c + 2 < pass_cols) top.offer(acc.z, ebase + c + 2);
          if (c + 3 < pass_cols) top.offer(acc.w, ebase + c + 3);
        }
      }
    }
    // every owner has pulled its rows from this CTA: its shared memory may take
    // the next expert group's loads, or be released when the CTA exits
    cluster_arrive_release();
    cluster_wait_acquire();
  }

  // ---------------- merge the segments, softmax, store ----------------
  merge_lane_groups(top, group);
  {
    const int t_local = static_cast<int>(r) + C * slot;
    const int64_t row = static_cast<int64_t>(tile) * BLOCK_M + t_local;
    if (group >= p.k) {  // every lane of the group holds the list: one entry per lane
      group_softmax_store(top, p.k, group, active, p.scores + row * p.k, p.ids + row * p.k);
      if (p.route.table != nullptr) group_route_count(p.route, top, p.k, group, active, row, p.E);
    } else if (active && seg == 0) {
      top.softmax_store(p.k, p.scores + row * p.k, p.ids + row * p.k);
      if (p.route.table != nullptr) route_count_row(p.route, top, p.k, row, p.E);
    }
  }
  if (clock_cta) record_launch_clock(p.clock, t0_ns, t0_clk);
}

}  // namespace tkg
