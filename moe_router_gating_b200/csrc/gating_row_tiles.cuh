// Persistent fused gating kernel: each CTA owns whole 128-token tiles.
//
// Per tile: logits[128, E] = hidden[128 rows, H] x gate[H, E] on the tensor
// cores (tcgen05.mma, bf16 in, fp32 accumulate in tensor memory), then per row
// top-k + softmax in registers; only scores and ids reach global memory.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: streams 64-wide K slices of the hidden tile
//               (K-major, 128-byte swizzle) and of the gate (MN-major,
//               128-byte swizzle, 64-expert boxes) through an S-stage ring.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma (4 per
//               stage, K=16 each) and commits stage releases / tile completion.
//   warps 2..5  epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 (one token
//               row per thread), keeps a running top-k, applies the softmax and
//               stores.  The accumulator is double-buffered in tensor memory so
//               the epilogue of tile i overlaps the MMAs of tile i+1.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "topk_epilogue.cuh"

namespace tkg {

constexpr int BLOCK_M = 128;                            // tokens per tile = TMEM lanes
constexpr int BLOCK_K = 64;                             // bf16 per 128-byte swizzle row
constexpr int UMMA_K = 16;                              // K per tcgen05.mma (kind::f16)
constexpr int A_STAGE_BYTES = BLOCK_M * BLOCK_K * 2;    // 16 KB hidden slice
constexpr int B_BOX_N = 64;                             // experts per gate box
constexpr int B_BOX_BYTES = BLOCK_K * B_BOX_N * 2;      // 8 KB gate box
constexpr int NUM_EPI_WARPS = 4;
constexpr int ROW_TILE_THREADS = 64 + NUM_EPI_WARPS * 32;

struct RowTileParams {
  int32_t T, H, E, k;
  int32_t n_pad;        // MMA N (E rounded up to 16)
  int32_t acc_stride;   // TMEM columns between the two accumulator buffers
  int32_t num_tiles;
  int32_t k_blocks;
  int32_t stages;
  int32_t b_boxes;      // ceil(n_pad / 64) gate boxes per stage
  uint32_t tmem_cols;
  uint64_t timeout_ns;
  float* scores;
  int32_t* ids;
  uint32_t* err_word;
};

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

template <int KMAX>
__global__ void __launch_bounds__(ROW_TILE_THREADS, 1)
    gating_row_tiles_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                            const RowTileParams p) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align_1024(smem_dyn);
  uint8_t* sA = smem;
  uint8_t* sB = smem + p.stages * A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + p.stages * p.b_boxes * B_BOX_BYTES);
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], NUM_EPI_WARPS * 32);
    }
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
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_x = l2_policy_evict_first();  // hidden: streamed once
      const uint64_t pol_w = l2_policy_evict_last();   // gate: re-read by every tile
      const uint32_t stage_tx = A_STAGE_BYTES + p.b_boxes * B_BOX_BYTES;
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns, ERR_WAIT_PRODUCER, p.err_word)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], stage_tx);
          tma_load_2d(sA + stage * A_STAGE_BYTES, &map_x, &full[stage], kb * BLOCK_K, tile * BLOCK_M, pol_x);
          for (int j = 0; j < p.b_boxes; ++j)
            tma_load_2d(sB + (stage * p.b_boxes + j) * B_BOX_BYTES, &map_w, &full[stage], j * B_BOX_N,
                        kb * BLOCK_K, pol_w);
          ++issued;
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Every load this thread issued lands before the CTA may exit.
      const int pending = issued < p.stages ? issued : p.stages;
      for (int n = 0; n < pending; ++n) {
        if (stage == 0) {
          stage = p.stages - 1;
          phase ^= 1;
        } else {
          --stage;
        }
        mbar_wait(&full[stage], phase, nullptr, p.timeout_ns, ERR_WAIT_DRAIN, p.err_word);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16_f32(BLOCK_M, p.n_pad, false, true);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local) {
        const uint32_t buf = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&acc_empty[buf], acc_phase ^ 1, abort_flag, p.timeout_ns, ERR_WAIT_MMA, p.err_word)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + buf * p.acc_stride;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.timeout_ns, ERR_WAIT_MMA, p.err_word)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * p.b_boxes * B_BOX_BYTES);
#pragma unroll
          for (int kk = 0; kk < BLOCK_K / UMMA_K; ++kk)
            umma_bf16(d_tmem, a_desc_k_slice(a_addr, kk), b_desc_k_slice(b_addr, kk), idesc, (kb | kk) != 0);
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit(&acc_full[buf]);
      }
      // Every MMA this thread issued completes before tensor memory is freed.
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.timeout_ns, ERR_WAIT_DRAIN, p.err_word);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;  // TMEM lanes this warp may access
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    int local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const uint32_t buf = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      bool ok = mbar_wait(&acc_full[buf], acc_phase, abort_flag, p.timeout_ns, ERR_WAIT_EPILOGUE, p.err_word);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after_sync();

      RowTopK<KMAX> top;
      top.reset();
      const uint32_t acc_addr = lane_base + buf * p.acc_stride;
      for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32(acc_addr + c0, r);
        tmem_ld_wait();
        if (c0 + 32 <= p.E) {
#pragma unroll
          for (int j = 0; j < 32; ++j) top.offer(__uint_as_float(r[j]), c0 + j);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < p.E) top.offer(__uint_as_float(r[j]), c0 + j);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&acc_empty[buf]);  // accumulator buffer may be overwritten

      const int64_t row = static_cast<int64_t>(tile) * BLOCK_M + quad * 32 + lane;
      if (row < p.T) top.softmax_store(p.k, p.scores + row * p.k, p.ids + row * p.k);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace tkg
