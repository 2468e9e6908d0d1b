// Fused gating for a handful of tokens on the CUDA cores, every SM streaming its
// own block of the gate matrix.
//
// A decode step's router reads the whole gate (H x E bf16: 3.67 MB at H = 7168,
// E = 256) for one to a few tokens.  That is a matrix-vector product: its time
// is the time to bring the gate in -- from all SMs at once -- plus the fixed
// costs of the launch and of combining the pieces, and tensor cores do not
// shorten either.  CTA (eb, hb) of a grid of e_blocks x h_blocks owns the 32
// experts [32 eb, 32 eb + 32) and the rows [h0, h1) of H:
//
//   1. it stages the tokens' hidden values of its rows in shared memory (fp32),
//      loads its gate block with 16-byte loads of 8 experts (a batch of up to
//      eight rows per thread in flight at once) and accumulates
//      partial[t][e] = sum over its rows h of hidden[t][h] * gate[h][e] in fp32
//      (the product of two bf16 values is exact in fp32);
//   2. it adds its threads' partials in a fixed order (a shuffle tree inside
//      each warp, then the warps 0..7 in turn) and stores the block's T x 32
//      partial logits to the workspace;
//   3. it counts itself on a workspace counter.  The CTA that arrives last
//      copies all partials into its shared memory (bulk copies), adds the
//      h_blocks partials of every logit in the order hb = 0, 1, ... -- so a
//      logit does not depend on which CTA came last -- and one warp per token
//      selects the k largest (ties to the lower expert index, the lane lists
//      merged by shuffles), applies the softmax over them and stores.
//
// No CTA waits for another: the last one finds every other block's partials
// stored (each CTA counts itself with a release after its stores, the count
// that finds all others there is an acquire).  The last CTA sets the counter
// back to zero, so it is zero between launches.
//
// The selection and softmax are those of the other gating kernels (the naive
// form on the chenxutan.com page "TileKernels 深度解析", section 4.1:
// logits = hidden_states @ gate_weight, the top k of each row, the softmax of
// those k values); only the order of the fp32 additions differs.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"
#include "topk_epilogue.cuh"
#include "topk_merge.cuh"

namespace tkg {

constexpr int FEW_THREADS = 256;
constexpr int FEW_WARPS = FEW_THREADS / 32;
constexpr int FEW_MAX_TOKENS = 4;   // tokens per launch of this kernel (from 4 on, split-H is as fast)
constexpr int FEW_EXPERTS = 32;     // experts per CTA: four 16-byte slots of 8
constexpr int FEW_MAX_EXPERTS = 256;  // E of a few-token call: at most 8 experts per lane in the selection
constexpr int FEW_ROW_GROUPS = FEW_THREADS / 4;  // threads sharing a slot: rows r, r + 64, ...
constexpr int FEW_BATCH = 8;        // gate rows per thread in flight
constexpr int FEW_COPY_CHUNK = 32768;  // bytes per bulk copy of the partials

struct FewTokenParams {
  const uint16_t* hidden;  // bf16 bits [T, H]
  const uint16_t* gate;    // bf16 bits [H, E]
  int32_t T, H, E, k;
  int32_t e_blocks;        // ceil(E / 32)
  int32_t h_blocks;        // CTAs per expert block, each owning h_rows rows of H (the last one fewer)
  int32_t h_rows;          // a multiple of 8
  int32_t e_pad;           // 32 * e_blocks: floats per partial row
  uint32_t* counter;       // workspace: CTAs done in this launch (zero between launches)
  float* part;             // workspace: [h_blocks][T][e_pad] partial logits
  float* scores;           // [T, k]
  int32_t* ids;            // [T, k]
  float* logits;           // optional [T, E]: every summed logit (verification)
  uint32_t* err_word;
  uint64_t timeout_ns;
  uint64_t* clock;
};

// Shared-memory layout (bytes from the dynamic base): the mbarrier and the
// last-arriver flag, the staged hidden values, the warps' sums, the copied
// partials and the summed logits.
struct FewTokenSmem {
  int32_t xs, red, parts, sums, total;
};

__host__ __device__ inline FewTokenSmem few_token_smem(int T, int h_rows, int h_blocks, int e_pad) {
  FewTokenSmem s;
  s.xs = 128;
  s.red = s.xs + (T * h_rows * 4 + 127) / 128 * 128;
  s.parts = s.red + FEW_WARPS * T * FEW_EXPERTS * 4;
  s.sums = s.parts + (h_blocks * T * e_pad * 4 + 127) / 128 * 128;
  s.total = s.sums + T * e_pad * 4;
  return s;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// the two bf16 values of a 32-bit word as fp32 (element 0 in the low half)
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int KMAX>
__global__ void __launch_bounds__(FEW_THREADS, 1) gating_few_tokens_kernel(const FewTokenParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint64_t t0_ns = globaltimer_ns();
  const uint64_t t0_clk = sm_clock64();
  const int tid = static_cast<int>(threadIdx.x);
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int T = p.T;
  const FewTokenSmem lay = few_token_smem(T, p.h_rows, p.h_blocks, p.e_pad);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  int* last_flag = reinterpret_cast<int*>(smem + 64);
  float* xs = reinterpret_cast<float*>(smem + lay.xs);      // [T][h_rows]
  float* red = reinterpret_cast<float*>(smem + lay.red);    // [warps][T][32]
  float* parts = reinterpret_cast<float*>(smem + lay.parts);  // [h_blocks][T][e_pad]
  float* sums = reinterpret_cast<float*>(smem + lay.sums);  // [T][e_pad]

  const int eb = static_cast<int>(blockIdx.x) % p.e_blocks;
  const int hb = static_cast<int>(blockIdx.x) / p.e_blocks;
  const int h0 = hb * p.h_rows;
  const int rows = min(p.h_rows, p.H - h0);  // > 0 and a multiple of 8 (the planner's blocks)
  const int slot = tid & 3;
  const int rg = tid >> 2;
  const int e_lo = eb * FEW_EXPERTS + slot * 8;
  const bool slot_on = e_lo < p.E;  // E % 8 == 0: a slot lies wholly inside E or past it
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  // inputs may come from the previous kernel in the stream
  griddep_wait();

  // first batch of gate rows in flight before the hidden values are staged
  const uint16_t* gp = p.gate + static_cast<int64_t>(h0 + rg) * p.E + e_lo;
  const int64_t batch_step = static_cast<int64_t>(FEW_ROW_GROUPS) * p.E;
  uint4 g[FEW_BATCH];
#pragma unroll
  for (int i = 0; i < FEW_BATCH; ++i) {
    const int r = rg + FEW_ROW_GROUPS * i;
    g[i] = (slot_on && r < rows) ? ldg_nc_v4(gp + i * batch_step) : make_uint4(0u, 0u, 0u, 0u);
  }
  {
    const int chunks = rows >> 3;  // 16-byte chunks of a token's row slice
    for (int q = tid; q < T * chunks; q += FEW_THREADS) {
      const int t = q / chunks;
      const int c = q - t * chunks;
      // the token's row slice inside hidden and inside the staging area
      if (!TK_CHECK(h0 + 8 * c + 8 <= p.H && (t * p.h_rows + 8 * c + 8) * 4 <= lay.red - lay.xs, p.err_word)) break;
      const uint4 v = ldg_nc_v4(p.hidden + static_cast<int64_t>(t) * p.H + h0 + 8 * c);
      float4* dst = reinterpret_cast<float4*>(xs + t * p.h_rows + 8 * c);
      dst[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
      dst[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
  }
  __syncthreads();

  float acc[FEW_MAX_TOKENS][8];
#pragma unroll
  for (int t = 0; t < FEW_MAX_TOKENS; ++t)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[t][j] = 0.0f;

  for (int r0 = 0;;) {
#pragma unroll
    for (int i = 0; i < FEW_BATCH; ++i) {
      const int r = r0 + rg + FEW_ROW_GROUPS * i;
      if (r < rows) {
        const float w[8] = {bf16_lo(g[i].x), bf16_hi(g[i].x), bf16_lo(g[i].y), bf16_hi(g[i].y),
                            bf16_lo(g[i].z), bf16_hi(g[i].z), bf16_lo(g[i].w), bf16_hi(g[i].w)};
#pragma unroll
        for (int t = 0; t < FEW_MAX_TOKENS; ++t) {
          if (t < T) {
            const float x = xs[t * p.h_rows + r];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[t][j] = fmaf(x, w[j], acc[t][j]);
          }
        }
      }
    }
    r0 += FEW_ROW_GROUPS * FEW_BATCH;
    if (r0 >= rows) break;
#pragma unroll
    for (int i = 0; i < FEW_BATCH; ++i) {
      const int r = r0 + rg + FEW_ROW_GROUPS * i;
      g[i] = (slot_on && r < rows) ? ldg_nc_v4(gp + (static_cast<int64_t>(r0) * p.E + i * batch_step))
                                   : make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // the eight row groups of a warp that share a slot: lanes slot, slot + 4, ..., added as a tree
#pragma unroll
  for (int t = 0; t < FEW_MAX_TOKENS; ++t) {
    if (t < T) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = acc[t][j];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        acc[t][j] = v;
      }
    }
  }
  if (lane < 4) {
#pragma unroll
    for (int t = 0; t < FEW_MAX_TOKENS; ++t) {
      if (t < T) {
        float4* dst = reinterpret_cast<float4*>(red + (warp * T + t) * FEW_EXPERTS + slot * 8);
        dst[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
        dst[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
      }
    }
  }
  __syncthreads();
  for (int q = tid; q < T * FEW_EXPERTS; q += FEW_THREADS) {
    const int t = q / FEW_EXPERTS;
    const int e = q - t * FEW_EXPERTS;
    float s = red[t * FEW_EXPERTS + e];
#pragma unroll
    for (int w = 1; w < FEW_WARPS; ++w) s += red[(w * T + t) * FEW_EXPERTS + e];
    if (!TK_CHECK(hb < p.h_blocks && eb * FEW_EXPERTS + e < p.e_pad, p.err_word)) break;
    p.part[(static_cast<int64_t>(hb) * T + t) * p.e_pad + eb * FEW_EXPERTS + e] = s;
  }

  // count this CTA done; the last one combines.  The barrier orders every
  // thread's partial stores before thread 0's arrival, whose release (gpu
  // scope, cumulative) publishes them; its acquire lets the last CTA read
  // the other CTAs' partials.
  __syncthreads();
  const uint32_t num_ctas = static_cast<uint32_t>(p.e_blocks * p.h_blocks);
  if (tid == 0) {
    const uint32_t before = atom_add_acq_rel_gpu(p.counter, 1u);
    const int last = before == num_ctas - 1;
    *last_flag = last;
    if (last) {
      *p.counter = 0u;  // every CTA of this launch has counted itself
      fence_proxy_async_global();  // the partials were stored by ordinary stores; the copies read them asynchronously
      uint32_t total = static_cast<uint32_t>(p.h_blocks * T * p.e_pad * 4);
      // the partials fit the shared-memory area they are copied to (else: no copy, the arrival alone)
      if (!TK_CHECK(total <= static_cast<uint32_t>(lay.sums - lay.parts), p.err_word)) total = 0;
      mbar_arrive_expect_tx(bar, total);
      for (uint32_t off = 0; off < total; off += FEW_COPY_CHUNK) {
        const uint32_t n = total - off < static_cast<uint32_t>(FEW_COPY_CHUNK) ? total - off
                                                                               : static_cast<uint32_t>(FEW_COPY_CHUNK);
        bulk_load_g2s(reinterpret_cast<uint8_t*>(parts) + off, reinterpret_cast<const uint8_t*>(p.part) + off, n, bar);
      }
    }
  }
  __syncthreads();
  if (!*last_flag) return;

  int abort_flag = 0;
  if (!mbar_wait(bar, 0, &abort_flag, p.timeout_ns, ERR_WAIT_EPILOGUE, p.err_word)) {
    // the copies land before the CTA may exit
    mbar_wait(bar, 0, nullptr, DRAIN_TIMEOUT_NS, ERR_WAIT_DRAIN, p.err_word);
    return;
  }
  const int part_stride = T * p.e_pad;  // floats from one H range's partial to the next
  for (int q = tid; q < T * p.E; q += FEW_THREADS) {
    const int t = q / p.E;
    const int e = q - t * p.E;
    const float* src = parts + t * p.e_pad + e;
    // added in the order of the H ranges; eight loads issued ahead of their additions
    float s = src[0];
    int h = 1;
    for (; h + 8 <= p.h_blocks; h += 8) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = src[(h + j) * part_stride];
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[j];
    }
    for (; h < p.h_blocks; ++h) s += src[h * part_stride];
    sums[t * p.e_pad + e] = s;
    if (p.logits != nullptr) p.logits[static_cast<int64_t>(t) * p.E + e] = s;
  }
  __syncthreads();

  // one warp per token: lane l offers its run of experts in increasing order,
  // then the 32 lane lists are merged
  const int per_lane = (p.E + 31) >> 5;
  for (int t = warp; t < T; t += FEW_WARPS) {
    RowTopK<KMAX> top;
    top.reset();
    const int e_begin = lane * per_lane;
    const int e_end = min(p.E, e_begin + per_lane);
    float v[FEW_MAX_EXPERTS / 32];  // the lane's values, loaded before its offers
#pragma unroll
    for (int j = 0; j < FEW_MAX_EXPERTS / 32; ++j) v[j] = e_begin + j < e_end ? sums[t * p.e_pad + e_begin + j] : 0.0f;
#pragma unroll
    for (int j = 0; j < FEW_MAX_EXPERTS / 32; ++j)
      if (e_begin + j < e_end) top.offer(v[j], e_begin + j);
    merge_lane_groups(top, 32);
    group_softmax_store(top, p.k, 32, true, p.scores + static_cast<int64_t>(t) * p.k,
                        p.ids + static_cast<int64_t>(t) * p.k);
  }
  if (tid == 0 && p.clock != nullptr) record_launch_clock(p.clock, t0_ns, t0_clk);
}

}  // namespace tkg
