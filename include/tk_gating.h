/*
 * tk_gating.h -- fused MoE top-k gating on NVIDIA B200 (sm_100a), C ABI.
 *
 * The operation (chenxutan.com, "TileKernels 深度解析", section 4.1 "MoE
 * Gating"): the router's three-step naive form
 *
 *     logits          = hidden_states @ gate_weight        [T,H] x [H,E]
 *     topk_vals, ids  = topk(logits, k)                     k largest per token
 *     scores          = softmax(topk_vals) over the k values
 *
 * replaced by one kernel launch in which the logits never leave the chip
 * (tensor memory and registers only; the page's "no write-back of
 * intermediates to global memory").
 *
 * Semantics fixed by this library where the page is silent:
 *   - logits accumulate in fp32 from bf16 inputs (no bf16 rounding of logits);
 *   - ranking order is logit descending, then expert index ascending (equal
 *     logits go to the lower expert index; -0 and +0 compare equal);
 *   - ids[t, 0..k-1] are in rank order, scores[t, 0] >= scores[t, 1] >= ...;
 *   - scores[t, j] = exp(v_j - v_0) / sum_i exp(v_i - v_0), fp32.
 *
 * Conventions for every entry point below:
 *   - Pointers marked "device" are CUDA global-memory addresses on the current
 *     device; the caller allocates and owns every buffer.  The library keeps no
 *     per-call state.  Only tk_gating_route allocates device memory: a
 *     stream-ordered workspace that it frees on the same stream.
 *     tk_gating_fused_topk_route uses a workspace that the caller owns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous: they return once the work is enqueued.  Launch
 *     failures return TK_ERR_CUDA; faults inside a kernel surface at the
 *     caller's next synchronisation.
 *   - Invalid arguments are rejected before any CUDA call; nothing is written.
 *   - There is no CPU fallback: without an sm_100 device every compute entry
 *     point returns TK_ERR_UNSUPPORTED or TK_ERR_CUDA.
 */
#ifndef TK_GATING_H
#define TK_GATING_H

#include <stdint.h>

#if defined(__GNUC__)
#define TK_API __attribute__((visibility("default")))
#else
#define TK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TK_OK = 0,
  TK_ERR_INVALID_ARG = -1,    /* null pointer, negative size, k out of [1, E], ... */
  TK_ERR_UNSUPPORTED = -2,    /* valid request outside what the kernels handle */
  TK_ERR_ALIGNMENT = -3,      /* a pointer is not 16-byte aligned */
  TK_ERR_CUDA = -4,           /* a CUDA runtime/driver call failed */
  TK_ERR_DEVICE_TIMEOUT = -5  /* a kernel's bounded wait expired (device error word set) */
} tk_status;

/* Limits of the fused kernels. */
#define TK_GATING_MAX_EXPERTS 1024
#define TK_GATING_MAX_TOPK 32

/*
 * tk_gating_fused_topk -- the fused gating operator.
 *
 *   hidden       device, bf16 [T, H] row-major (token t at hidden + t*H).
 *   gate_weight  device, bf16 [H, E] row-major (the [H,E] orientation of
 *                `hidden_states @ gate_weight`; expert e is column e).
 *   T            tokens, T >= 0.  T == 0 returns TK_OK and launches nothing.
 *   H            hidden size, H >= 8 and H % 8 == 0 (16-byte row pitch).
 *   E            experts, 16 <= E <= 1024 and E % 8 == 0.
 *   k            experts kept per token, 1 <= k <= min(E, 32).
 *   scores       device, out fp32 [T, k] row-major.
 *   ids          device, out int32 [T, k] row-major.
 *   stream       cudaStream_t (void*), may be NULL.
 *
 * Errors:
 *   TK_ERR_INVALID_ARG   T < 0, H < 1, E < 1, k < 1, k > E, or a null pointer
 *                        when T > 0;
 *   TK_ERR_UNSUPPORTED   H or E not a multiple of 8, E < 16, E > 1024, k > 32,
 *                        T >= 2^31 - 128, or the current device is not sm_100;
 *   TK_ERR_ALIGNMENT     a pointer is not 16-byte aligned;
 *   TK_ERR_CUDA          a CUDA call (device query, descriptor encode, launch)
 *                        failed.
 * Size checks come first, so an invalid size is reported even with null
 * pointers; T == 0 with valid sizes returns TK_OK before pointers are looked at.
 */
TK_API tk_status tk_gating_fused_topk(const void* hidden, const void* gate_weight, int64_t T, int64_t H, int64_t E,
                               int32_t k, float* scores, int32_t* ids, void* stream);

/*
 * tk_gating_fused_topk_host -- the same operator for inputs and outputs that
 * live in host memory (an end-to-end call).  On `stream` it copies hidden from
 * host to the caller's device staging buffer, runs the fused kernel, and copies
 * scores and ids back to host.  The gate stays device-resident (model weights).
 *
 *   hidden_host  host, bf16 [T, H]; page-locked memory makes the copy async.
 *   gate_weight  device, bf16 [H, E].
 *   scores_host  host, out fp32 [T, k].   ids_host  host, out int32 [T, k].
 *   hidden_dev   device staging, bf16 [T, H].
 *   scores_dev   device staging, fp32 [T, k].   ids_dev  device staging, int32 [T, k].
 *
 * Host buffers must stay valid until the stream reaches this point.  Same
 * errors as tk_gating_fused_topk, plus TK_ERR_INVALID_ARG for null host
 * pointers.
 */
TK_API tk_status tk_gating_fused_topk_host(const void* hidden_host, const void* gate_weight, int64_t T, int64_t H,
                                    int64_t E, int32_t k, float* scores_host, int32_t* ids_host, void* hidden_dev,
                                    float* scores_dev, int32_t* ids_dev, void* stream);

/*
 * tk_gating_fused_topk_fp8 -- the fused gating operator on FP8 (E4M3) inputs.
 *
 * The gating of section 4.1 on inputs quantized as the page's section 4.3
 * "Quantization" describes (FP8 E4M3 values with a per-token scale, its
 * per_token_quantize).  A tensor-core FP8 product needs both operands in FP8,
 * so the gate is quantized too, with one scale per expert:
 *
 *   hidden[t, h] = hidden_scale[t] * e4m3(hidden_q[t, h])
 *   gate[h, e]   = gate_scale[e]   * e4m3(gate_q[e, h])
 *   logits[t, e] = (sum_h e4m3(hidden_q[t, h]) * e4m3(gate_q[e, h])) * gate_scale[e] * hidden_scale[t]
 *
 * The products are exact and summed in fp32 on the tensor cores
 * (tcgen05.mma kind::f8f6f4); the two scales are applied in fp32 in that
 * order; ranking, top-k and softmax as tk_gating_fused_topk.
 *
 *   hidden_q      device, E4M3 bytes [T, H] row-major.
 *   hidden_scale  device, fp32 [T].
 *   gate_q        device, E4M3 bytes [E, H] row-major: expert-major, each
 *                 expert's H values contiguous (the layout of a quantized
 *                 [E, H] linear weight with one scale per row).
 *   gate_scale    device, fp32 [E].
 *   T, E, k, scores, ids, stream  as tk_gating_fused_topk;  H % 16 == 0.
 *
 * Errors as tk_gating_fused_topk (every pointer, the scales included, must be
 * 16-byte aligned; H not a multiple of 16 is TK_ERR_UNSUPPORTED).  The launch is
 * the one tk_gating_make_plan gives for (T, H / 2, E, k): a K slice of 128 FP8
 * values takes the shared memory of 64 bf16 values.
 */
TK_API tk_status tk_gating_fused_topk_fp8(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                          const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k,
                                          float* scores, int32_t* ids, void* stream);

/*
 * tk_gating_fused_topk_logits / tk_gating_fused_topk_fp8_logits -- the same
 * operators, which also store every logit their selection ranked.
 *
 * A verification aid for the logits step of section 4.1 (logits =
 * hidden_states @ gate_weight, here in fp32 on the tensor cores): the launch
 * is the one tk_gating_fused_topk (or _fp8) makes, the same kernels, whose
 * epilogue additionally writes each fp32 logit it offers to the selection
 * (FP8: after both scales).  scores and ids are bitwise the ones the plain
 * call returns.  Not for production use: it writes T x E x 4 bytes more.
 *
 *   logits   device, out fp32 [T, E] row-major, 16-byte aligned.
 *   the other arguments as tk_gating_fused_topk (or _fp8).
 *
 * Errors as tk_gating_fused_topk (or _fp8); TK_ERR_INVALID_ARG for a null
 * logits when T > 0, TK_ERR_ALIGNMENT when it is not 16-byte aligned.
 */
TK_API tk_status tk_gating_fused_topk_logits(const void* hidden, const void* gate_weight, int64_t T, int64_t H,
                                             int64_t E, int32_t k, float* scores, int32_t* ids, float* logits,
                                             void* stream);
TK_API tk_status tk_gating_fused_topk_fp8_logits(const void* hidden_q, const float* hidden_scale,
                                                 const void* gate_q, const float* gate_scale, int64_t T, int64_t H,
                                                 int64_t E, int32_t k, float* scores, int32_t* ids, float* logits,
                                                 void* stream);

/* Kernel variants chosen by the planner. */
typedef enum {
  TK_VARIANT_NONE = 0,        /* T == 0: nothing to launch */
  TK_VARIANT_ROW_TILES = 1,   /* persistent: each CTA owns whole 128-token tiles */
  TK_VARIANT_SPLIT_H = 2,     /* a cluster of CTAs splits H for one tile, DSMEM reduction */
  TK_VARIANT_ROW_PAIRS = 3,   /* persistent CTA pairs (tcgen05 cta_group::2), 256-token tiles */
  TK_VARIANT_FEW_TOKENS = 4   /* workspace entry points, T <= 4: CUDA-core blocks of H x 32 experts,
                                 partial logits combined by the CTA that finishes last */
} tk_variant;

/* The launch the library makes for a problem (host logic, no GPU needed). */
typedef struct {
  int32_t variant;      /* tk_variant */
  int32_t block_m;      /* tokens per tile */
  int32_t n_pad;        /* MMA N over all experts: E rounded up to a multiple of 16 (CTA pairs: of
                           128); one MMA per chunk of up to 256 experts and K step */
  int32_t num_tiles;    /* full tiles of block_m tokens (all of T unless num_half_tiles > 0) */
  int32_t k_blocks;     /* ceil(H / 64) */
  int32_t split_h;      /* CTAs sharing one tile's H range (1 = none) */
  int32_t stages;       /* shared-memory ring depth, in stages of slices_per_stage K slices */
  int32_t grid;         /* CTAs launched */
  int32_t cluster;      /* CTAs per cluster */
  int32_t threads;      /* threads per CTA */
  int32_t smem_bytes;   /* dynamic shared memory per CTA */
  int32_t tmem_cols;    /* tensor-memory columns allocated per CTA */
  int32_t num_half_tiles; /* CTA pairs: 128-token tiles after the full ones (balanced last round) */
  int32_t slices_per_stage; /* 64-wide K slices per ring stage */
  int32_t expert_groups;  /* groups of at most 512 experts, computed one after the other per tile (1 or 2) */
  int32_t num_split_tiles; /* workspace entry points: last-round 256-token tiles each split in H between two
                              CTA pairs, in place of the half tiles (0: none) */
  int32_t split_k_block;   /* the K slice (of 64) at which a split tile's H range is cut */
  int32_t h_rows;          /* TK_VARIANT_FEW_TOKENS: rows of H per CTA (split_h CTAs per block of 32
                              experts, n_pad / 32 blocks; block_m = T) */
} tk_gating_plan;

/*
 * tk_gating_make_plan -- fill *plan with the launch tk_gating_fused_topk makes
 * for (T, H, E, k) on a device with `num_sms` SMs whose clusters fit like a
 * B200's (of 148 SMs, 74 / 33 / 15 / 7 clusters of 2 / 4 / 8 / 16 CTAs run at
 * once; scaled by num_sms / 148).  The launch itself uses the current device's
 * measured cluster capacities, so on other parts the cluster size may differ.
 * Validates like tk_gating_fused_topk (pointers excepted).  Makes no CUDA call.
 */
TK_API tk_status tk_gating_make_plan(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms, tk_gating_plan* plan);

/*
 * tk_gating_fused_topk_ws -- tk_gating_fused_topk with a caller-owned device
 * workspace, which lets a call of a few tokens spread over every SM and a
 * many-token launch end its last round sooner.
 *
 * The operation, outputs and errors are those of tk_gating_fused_topk
 * (section 4.1, "MoE Gating"); only the schedule differs, in two cases.
 *
 * 1 <= T <= 4 and E <= 256 (decode; plan variant TK_VARIANT_FEW_TOKENS): the
 * launch runs about one CTA per SM, each owning a block of 32 experts and a
 * range of H rows.  A CTA accumulates its block's partial logits on the CUDA
 * cores (fp32, each bf16 product exact) and stores them to the workspace; the
 * CTA that finishes last adds the partials of every logit in the order of the
 * H ranges, selects, applies the softmax and stores.  No CTA waits for
 * another.  The logits are fp32 sums in another association than the plain
 * call's, so selections agree wherever the k-th and (k+1)-th logits are not
 * within fp32 rounding.  bf16 only (the FP8 entry point keeps its plain plan
 * for these T).
 *
 * Many tokens: where the plan without workspace ends with a round of 128-token "half" tiles
 * on CTA pairs (many tokens, 64 < E <= 256, k <= 8, and long tiles: at least
 * 96 K slices, i.e. H >= 6144 bf16 or H >= 12288 FP8 values), this call instead cuts
 * each of the last round's 256-token tiles in H between two CTA pairs: the
 * first accumulates H slices [0, split_k_block) of the tile and stores its
 * fp32 accumulator rows to the workspace, the second accumulates the rest,
 * adds the stored rows to its own (first half + second half, fp32) and selects,
 * applies the softmax and stores as tk_gating_fused_topk does.  A split tile
 * costs about half of a full tile where a half tile costs ~0.9.  The logits
 * of those rows are therefore fp32 sums in a different association; selections
 * agree wherever the k-th and (k+1)-th logits are not within fp32 rounding.
 * Elsewhere the launch is tk_gating_fused_topk's and the workspace untouched.
 *
 *   workspace        device, 16-byte aligned, at least the bytes that
 *                    tk_gating_workspace_bytes (or tk_gating_make_plan_ws)
 *                    gives for this call (9.1 MB at T = 65536, E = 256,
 *                    k = 8; 74.0 KB at T = 4, H = 7168, E = 256; on a
 *                    B200); may be NULL when that is 0.  It starts with
 *                    flags (8 bytes per split tile, rounded up to 256) or a
 *                    counter (the few-token case, 256 bytes) that must be
 *                    zero before the first call: zero the workspace once
 *                    after allocating it; every call leaves them zero, so
 *                    calls in order on one stream may share a workspace
 *                    whatever their sizes (one large enough for each).  Calls
 *                    that may run at the same time need workspaces of their
 *                    own.  After a call that reported an expired wait
 *                    (tk_gating_device_error), zero it again.
 *   workspace_bytes  its size.
 *   the other arguments as tk_gating_fused_topk.
 *
 * The second half's pair waits (bounded, as every wait in the kernels) for
 * the first half's rows; both are CTAs of the same launch, which fits one
 * wave.  Errors: those of tk_gating_fused_topk, and TK_ERR_INVALID_ARG when
 * the workspace is NULL or smaller than needed (or workspace_bytes < 0),
 * TK_ERR_ALIGNMENT when it is not 16-byte aligned.  Allocates nothing.
 */
TK_API tk_status tk_gating_fused_topk_ws(const void* hidden, const void* gate_weight, int64_t T, int64_t H,
                                         int64_t E, int32_t k, float* scores, int32_t* ids, void* workspace,
                                         int64_t workspace_bytes, void* stream);

/*
 * tk_gating_fused_topk_fp8_ws -- tk_gating_fused_topk_fp8 with a workspace, as
 * tk_gating_fused_topk_ws: the stored first half is the unscaled fp32 sum of
 * E4M3 products; the second half's pair scales each summed logit by
 * gate_scale[e] and then hidden_scale[t], as tk_gating_fused_topk_fp8 does.
 */
TK_API tk_status tk_gating_fused_topk_fp8_ws(const void* hidden_q, const float* hidden_scale, const void* gate_q,
                                             const float* gate_scale, int64_t T, int64_t H, int64_t E, int32_t k,
                                             float* scores, int32_t* ids, void* workspace, int64_t workspace_bytes,
                                             void* stream);

/*
 * tk_gating_fused_topk_ws_logits -- tk_gating_fused_topk_ws that also stores
 * every logit its selection ranked into logits (device, fp32 [T, E], 16-byte
 * aligned), as tk_gating_fused_topk_logits does.  A verification aid.
 */
TK_API tk_status tk_gating_fused_topk_ws_logits(const void* hidden, const void* gate_weight, int64_t T, int64_t H,
                                                int64_t E, int32_t k, float* scores, int32_t* ids, float* logits,
                                                void* workspace, int64_t workspace_bytes, void* stream);

/*
 * tk_gating_make_plan_ws -- the launch tk_gating_fused_topk_ws makes for
 * (T, H, E, k) on a device like tk_gating_make_plan's, and the workspace bytes
 * it needs (0 when the launch is the one without workspace).  Makes no CUDA
 * call.  tk_gating_make_plan_fp8_ws: the same for tk_gating_fused_topk_fp8_ws
 * (H counts FP8 values; validated like that call).
 */
TK_API tk_status tk_gating_make_plan_ws(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms,
                                        tk_gating_plan* plan, int64_t* workspace_bytes);
TK_API tk_status tk_gating_make_plan_fp8_ws(int64_t T, int64_t H, int64_t E, int32_t k, int32_t num_sms,
                                            tk_gating_plan* plan, int64_t* workspace_bytes);

/*
 * tk_gating_workspace_bytes -- the workspace bytes tk_gating_fused_topk_ws
 * (fp8 = 0) or tk_gating_fused_topk_fp8_ws (fp8 != 0) needs for (T, H, E, k)
 * on the current device.  Validates the sizes like those calls.  Errors:
 * TK_ERR_INVALID_ARG for a null result pointer, the size errors, and
 * TK_ERR_CUDA / TK_ERR_UNSUPPORTED without an sm_100 device.
 */
TK_API tk_status tk_gating_workspace_bytes(int64_t T, int64_t H, int64_t E, int32_t k, int32_t fp8,
                                           int64_t* workspace_bytes);

/*
 * tk_gating_device_error -- read the device error word of the current device
 * into *word (0 = none), and clear it when `clear` is non-zero.  Bits: 0..4 a
 * bounded wait expired (producer, MMA, epilogue, drain, cluster); 5 an index
 * check failed and its access was skipped (only in the checked build,
 * libtk_gating_debug.so, compiled with TK_GATING_DEBUG); 6 the routing counts
 * taken by the gating disagreed with the ids (tk_gating_fused_topk_route
 * given a workspace that was not zero); 8 an expert-parallel
 * row address was not 16-byte aligned.  Synchronises the device.  Returns
 * TK_ERR_DEVICE_TIMEOUT when the word is non-zero, TK_OK otherwise.
 */
TK_API tk_status tk_gating_device_error(uint32_t* word, int32_t clear);

/*
 * tk_gating_clock_counters -- SM-clock record of the fused gating launches on
 * the current device.  The first CTA of every launch of tk_gating_fused_topk
 * (and of its variants) adds the SM clock cycles and the nanoseconds from its
 * start to its end, and 1, to three device counters; this call reads them into
 * *sm_cycles, *elapsed_ns and *launches, and zeroes them when `clear` is
 * non-zero.  sm_cycles / elapsed_ns is the mean SM clock (GHz) under the
 * launches' own load -- a measurement aid for timing.  Synchronises the
 * device.  TK_ERR_INVALID_ARG for a null pointer, TK_ERR_CUDA when a CUDA call
 * fails.  Counters of a device no gating call has run on read as zero.
 */
TK_API tk_status tk_gating_clock_counters(uint64_t* sm_cycles, uint64_t* elapsed_ns, uint64_t* launches,
                                          int32_t clear);

/*
 * tk_gating_set_wait_timeout_ns -- limit (nanoseconds) of every bounded wait in
 * the kernels launched afterwards from this process (default 1e9).  Values
 * below 1000 are rejected with TK_ERR_INVALID_ARG.
 */
TK_API tk_status tk_gating_set_wait_timeout_ns(uint64_t timeout_ns);

/*
 * ---------------------------------------------------------------------------
 * Routing metadata (the local part of MoE dispatch).
 *
 * The operation (chenxutan.com, "TileKernels 深度解析", section 4.2 "MoE
 * Routing"): dispatch sends every token to the experts its expert_ids row
 * names, and combine puts the experts' results back with the indices dispatch
 * returned.  Before any exchange, the T*k token-expert assignments have to be
 * grouped by expert.  For assignment s = t*k + j (token t, rank j) with expert
 * e = ids[s]:
 *
 *   offsets[e]       number of assignments to experts below e (exclusive
 *                    prefix sum of the per-expert counts); offsets[E] is the
 *                    number placed, so expert e owns positions
 *                    [offsets[e], offsets[e+1]);
 *   sorted_slots[p]  the assignment s at position p of the grouped order;
 *                    inside an expert the assignments keep ascending s (a
 *                    stable order: the result is unique and deterministic);
 *   slot_pos[s]      the position p of assignment s (the inverse of
 *                    sorted_slots; the page's dispatch_indices in this
 *                    library's reading).
 *
 * An id outside [0, E) is neither counted nor placed: its slot_pos is -1 and
 * offsets[E] falls short of T*k by the number of such ids; the positions
 * offsets[E] .. T*k-1 of sorted_slots are then not written.
 * ---------------------------------------------------------------------------
 */
#define TK_ROUTE_MAX_EXPERTS 1024

/* The launches tk_gating_route makes (host logic, no GPU needed). */
typedef struct {
  int32_t ctas;               /* CTAs of each kernel; 1 = a single kernel and no workspace */
  int32_t threads;            /* threads per CTA */
  int64_t warp_slots;         /* assignments per warp range (a multiple of 32) */
  int64_t workspace_bytes;    /* device workspace: ctas x round_up(E, 4) int32 counts, 0 when ctas == 1 */
  int32_t count_smem_bytes;   /* dynamic shared memory of the counting kernel */
  int32_t scatter_smem_bytes; /* dynamic shared memory of the placing kernel */
  int64_t fused_workspace_bytes; /* workspace of tk_gating_fused_topk_route: the counts table and a
                                    16-byte arrival counter (workspace_bytes + 16), 0 when ctas == 1 */
} tk_route_plan;

/*
 * tk_gating_route -- routing metadata of ids[T, k].
 *
 *   ids           device, int32 [T, k] row-major (for example the ids output
 *                 of tk_gating_fused_topk); read only.
 *   T, k          tokens (T >= 0) and assignments per token (k >= 1);
 *                 T * k < 2^31.
 *   E             experts, 1 <= E <= 1024.
 *   offsets       device, out int32 [E + 1].
 *   sorted_slots  device, out int32 [T * k].
 *   slot_pos      device, out int32 [T, k].
 *   stream        cudaStream_t (void*), may be NULL.
 *
 * Up to 4096 assignments: one kernel launch on `stream`, no workspace.
 * Beyond: two launches, the second a programmatic dependent launch of the
 * first, with a workspace of tk_route_plan.workspace_bytes (at most
 * 148 x 1024 x 4 bytes on a B200) that the call takes with cudaMallocAsync
 * from the device's default memory pool and releases with cudaFreeAsync after
 * the launches, both on `stream`.  T * k == 0 is valid: offsets is set to
 * zeros and ids, sorted_slots and slot_pos may then be NULL.
 *
 * Errors:
 *   TK_ERR_INVALID_ARG   T < 0, k < 1, E < 1, offsets NULL, or another
 *                        pointer NULL when T * k > 0;
 *   TK_ERR_UNSUPPORTED   E > 1024, T * k >= 2^31, or the device is not sm_100;
 *   TK_ERR_ALIGNMENT     a pointer is not 4-byte aligned;
 *   TK_ERR_CUDA          the workspace allocation or a launch failed.
 */
TK_API tk_status tk_gating_route(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                                 int32_t* sorted_slots, int32_t* slot_pos, void* stream);

/*
 * tk_gating_route_plan -- fill *plan with the launches tk_gating_route makes
 * for (T, k, E) on a device with `num_sms` SMs.  Validates sizes like
 * tk_gating_route.  Makes no CUDA call.
 */
TK_API tk_status tk_gating_route_plan(int64_t T, int32_t k, int32_t E, int32_t num_sms, tk_route_plan* plan);

/*
 * tk_gating_fused_topk_route -- tk_gating_fused_topk followed by
 * tk_gating_route of its ids, with the routing's counting step done by the
 * gating kernel: each selected (token, expert) assignment is added to a small
 * table of per-expert counts (atomic adds in global memory) as the gating
 * stores it (chenxutan.com, "TileKernels 深度解析", section 4.2 "MoE Routing":
 * the counts per expert that dispatch starts from, taken where the ids are
 * produced).  The placing kernel then reads the table instead of counting the
 * ids in a launch of its own.  Outputs, layouts and results are exactly those
 * of the two calls made one after the other.
 *
 *   hidden, gate_weight, T, H, E, k, scores, ids   as tk_gating_fused_topk.
 *   offsets, sorted_slots, slot_pos                as tk_gating_route
 *                                                  (4-byte aligned).
 *   workspace     device, at least tk_route_plan.fused_workspace_bytes
 *                 (tk_gating_route_plan of (T, k, E) on this device's SM
 *                 count), 16-byte aligned; may be NULL when that is 0.  It
 *                 must hold zeros when a call starts: zero it once after
 *                 allocating it; every call leaves the part it used zero
 *                 again, so one workspace serves any sequence of calls
 *                 issued in order (one stream).  Calls that overlap need
 *                 workspaces of their own.
 *   workspace_bytes  its size.
 *   stream        cudaStream_t (void*), may be NULL.
 *
 * Launches on `stream`: the gating kernel, then (up to 4096 assignments) the
 * routing's one-CTA kernel -- the table is then not used -- or the placing
 * kernel, launched as a programmatic dependent of the gating.  Allocates
 * nothing.
 *
 * The placing kernel checks the table against the ids it reads: a CTA whose
 * row of the table differs from its own count of its assignments (a workspace
 * that was not zero) sets bit 6 of the device error word
 * (tk_gating_device_error), and no position outside [0, T*k) is written; the
 * routing outputs of that call are then not valid.  Zero the workspace again
 * after bit 6 was reported (stale counts alone are cleared by the call itself,
 * a stale arrival counter in the last 16 bytes is not).
 *
 * Errors: those of tk_gating_fused_topk and of tk_gating_route, and
 *   TK_ERR_INVALID_ARG   workspace NULL or smaller than
 *                        tk_route_plan.fused_workspace_bytes while that is > 0;
 *   TK_ERR_ALIGNMENT     workspace not 16-byte aligned.
 */
TK_API tk_status tk_gating_fused_topk_route(const void* hidden, const void* gate_weight, int64_t T, int64_t H,
                                            int64_t E, int32_t k, float* scores, int32_t* ids, int32_t* offsets,
                                            int32_t* sorted_slots, int32_t* slot_pos, void* workspace,
                                            int64_t workspace_bytes, void* stream);

/*
 * tk_gating_route_static -- tk_gating_route without any allocation.
 *
 * The pages have no counterpart: this is a property of this library's
 * interface.  It is for callers that cannot let the library allocate device
 * memory: a process whose device memory is reserved up front by its own
 * allocator (a pool allocation could then fail in the middle of a run), or
 * code that must not enter the driver's allocator at all (growing a memory
 * pool maps new memory).  The result is the same as tk_gating_route's; the
 * counts table that tk_gating_route takes from cudaMallocAsync lives here in
 * a fixed device array of TK_ROUTE_STATIC_SCRATCH_BYTES, one per device.
 *
 *   Arguments, layouts and the other errors as tk_gating_route.
 *   TK_ERR_UNSUPPORTED also when the launch needs more scratch than the array
 *   holds (tk_route_plan.workspace_bytes > TK_ROUTE_STATIC_SCRATCH_BYTES):
 *   never for E <= 440 on a device of at most 148 SMs; for larger E while the
 *   plan's ctas x round_up(E, 4) x 4 bytes fit (E = 1024: up to 262144
 *   assignments).  Nothing is written then.
 *   TK_ERR_CUDA when the array's device address cannot be obtained.
 *
 * Set-up: the first call made with a device current looks up the array's
 * device address on that device (and loads the library's kernels there if
 * that has not happened yet); make that first call before any stream capture.
 * Calls that overlap on one device (issued to different streams, or from
 * different host threads, without ordering between them) share the one
 * array and race: order them, for example by issuing them to one stream.
 */
#define TK_ROUTE_STATIC_SCRATCH_BYTES (256 * 1024)
TK_API tk_status tk_gating_route_static(const int32_t* ids, int64_t T, int32_t k, int32_t E, int32_t* offsets,
                                        int32_t* sorted_slots, int32_t* slot_pos, void* stream);

/*
 * ---------------------------------------------------------------------------
 * Expert-parallel dispatch and combine.
 *
 * The operation (chenxutan.com, "TileKernels 深度解析", section 4.2 "MoE
 * Routing": fused_dispatch(tokens, expert_ids, num_experts, ep_group) sends
 * every token to the GPUs holding the experts its expert_ids row names;
 * fused_combine(expert_output, dispatch_indices, scores, ep_group) brings the
 * experts' results back and sums them weighted by the gating scores).  In an
 * expert-parallel group of R ranks, rank q holds experts [q*E/R, (q+1)*E/R).
 * Rank q's receive buffer holds, for each of its experts in ascending order,
 * for each source rank in ascending order, that source's rows for the expert
 * in ascending assignment order s = t*k + j.  The expert outputs are expected
 * in the same layout (one output row per received row).
 *
 * Both calls address the expert buffers through a device table of E row
 * addresses: rows[e] = the address of this source rank's first row for
 * expert e in the buffer of the rank that holds e (a local buffer, or another
 * GPU's buffer opened with tk_gating_ep_ipc_open).  Assignment s with expert
 * e = ids[s] at position p = slot_pos[s] of the expert-grouped order (offsets
 * and slot_pos from tk_gating_route) uses row rows[e] + (p - offsets[e]).  Dispatch stores each token row there; combine loads the
 * expert output rows from there (the receiver pulls, as the page's section 6
 * recommends), so the data crosses NVLink once and no all-to-all runs.
 * Ordering between ranks is the caller's: every rank's dispatch has to be
 * complete before the experts read the receive buffers, every expert output
 * before combine reads it.  A row address that is not 16-byte aligned is
 * skipped and sets bit 8 of the device error word (tk_gating_device_error).
 * ---------------------------------------------------------------------------
 */

/*
 * tk_gating_fused_dispatch -- copy every placed assignment's token row to
 * its row in the expert buffer.  Each token row is read once and stored to
 * each of its k destination rows.
 *
 *   tokens        device, bf16 [T, H] row-major, 16-byte aligned.
 *   T, H, k, E    tokens (T >= 0), hidden size (H % 8 == 0), experts per
 *                 token (1 <= k <= 32), experts (1 <= E <= 1024); T*k < 2^31.
 *   ids           device, int32 [T, k]: the experts (tk_gating_fused_topk).
 *   offsets       device, int32 [E + 1]     } tk_gating_route of ids
 *   slot_pos      device, int32 [T, k]      }   (assignments whose id is
 *                 outside [0, E) or whose slot_pos is -1 are not copied)
 *   rows          device, uint64 [E]: destination address of expert e's first
 *                 row for this rank (16-byte aligned; device or peer memory).
 *   stream        cudaStream_t (void*), may be NULL.
 *
 * Errors: TK_ERR_INVALID_ARG (negative sizes, k or E < 1, null pointers when
 * T > 0), TK_ERR_UNSUPPORTED (H % 8, k > 32, E > 1024, T*k >= 2^31),
 * TK_ERR_ALIGNMENT (tokens not 16-byte, rows not 8-byte, the int32 arrays
 * not 4-byte aligned), TK_ERR_CUDA (launch failure or no sm_100 device).
 * T == 0 returns TK_OK and launches nothing.
 */
TK_API tk_status tk_gating_fused_dispatch(const void* tokens, int64_t T, int64_t H, int32_t k, int32_t E,
                                          const int32_t* ids, const int32_t* offsets, const int32_t* slot_pos,
                                          const uint64_t* rows, void* stream);

/*
 * tk_gating_fused_combine -- out[t] = sum_j scores[t, j] * y(t, j), where
 * y(t, j) is the expert output row of assignment (t, j), in fp32 (fused
 * multiply-adds in rank order j = 0 .. k-1), rounded once to bf16.
 * Assignments whose id is outside [0, E) or whose slot_pos is -1 contribute
 * nothing.
 *
 *   rows          device, uint64 [E]: address of expert e's first output row
 *                 for this rank (the table dispatch used, pointing into the
 *                 expert output buffers).
 *   ids, offsets  as tk_gating_fused_dispatch;  slot_pos  device, int32 [T, k]
 *                 (tk_gating_route);  scores  device, fp32 [T, k].
 *   out           device, out bf16 [T, H], 16-byte aligned.
 *
 * Errors as tk_gating_fused_dispatch (out 16-byte aligned, scores 4-byte).
 */
TK_API tk_status tk_gating_fused_combine(const uint64_t* rows, int64_t T, int64_t H, int32_t k, int32_t E,
                                         const int32_t* ids, const int32_t* offsets, const int32_t* slot_pos,
                                         const float* scores, void* out, void* stream);

/*
 * tk_gating_ep_rows_table -- the row-address tables of source rank `rank`
 * from every rank's routing offsets (one small launch).
 *
 *   offsets_all   device, int32 [R, E + 1]: row s = rank s's tk_gating_route
 *                 offsets (gathered from every rank); rank s has
 *                 offsets_all[s, e+1] - offsets_all[s, e] assignments to e.
 *   R, E, rank    ranks (E % R == 0, E <= 1024), this rank (0 <= rank < R).
 *   bases         device, uint64 [R]: address of rank q's receive buffer, as
 *                 this process sees it (its own, or opened from a handle).
 *   out_bases     device, uint64 [R] or NULL: the same for the expert output
 *                 buffers (rows of the same layout).
 *   H             hidden size (row pitch H * 2 bytes).
 *   rows          device, out uint64 [E]: tk_gating_fused_dispatch's table.
 *   out_rows      device, out uint64 [E] or NULL: tk_gating_fused_combine's
 *                 table (from out_bases).
 *   recv_offsets  device, out int32 [E/R + 1]: the first row of each of this
 *                 rank's experts in its own receive buffer (and the total).
 *
 * Errors: TK_ERR_INVALID_ARG (R < 1, rank outside [0, R), null pointers),
 * TK_ERR_UNSUPPORTED (E % R != 0, E > 1024, H % 8), TK_ERR_ALIGNMENT,
 * TK_ERR_CUDA.
 */
TK_API tk_status tk_gating_ep_rows_table(const int32_t* offsets_all, int32_t R, int32_t E, int32_t rank,
                                         const uint64_t* bases, const uint64_t* out_bases, int64_t H, uint64_t* rows,
                                         uint64_t* out_rows, int32_t* recv_offsets, void* stream);

/*
 * Inter-process handles of device buffers, so that a rank can address
 * another rank's expert buffers (on another GPU over NVLink, or on the same
 * GPU).  tk_gating_ep_ipc_handle writes a handle of TK_EP_IPC_HANDLE_BYTES
 * bytes for the device pointer (the CUDA IPC handle of the allocation that
 * contains it, plus the offset into it); another process passes those bytes to
 * tk_gating_ep_ipc_open, which maps the allocation and returns the same
 * buffer's address in that process; tk_gating_ep_ipc_close(ptr, handle) unmaps
 * it.  The owner must keep the allocation alive while it is open elsewhere.
 * TK_ERR_INVALID_ARG for null arguments or a pointer that is not device
 * memory; TK_ERR_CUDA when the CUDA IPC call fails.
 */
#define TK_EP_IPC_HANDLE_BYTES 128
TK_API tk_status tk_gating_ep_ipc_handle(const void* dev_ptr, void* handle);
TK_API tk_status tk_gating_ep_ipc_open(const void* handle, void** dev_ptr);
TK_API tk_status tk_gating_ep_ipc_close(void* dev_ptr, const void* handle);

/* Static string for a status code. */
TK_API const char* tk_gating_status_string(tk_status status);

#ifdef __cplusplus
}
#endif

#endif /* TK_GATING_H */
