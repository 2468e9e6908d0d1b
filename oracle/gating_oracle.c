/*
 * CPU oracle for fused MoE top-k gating.  TEST INFRASTRUCTURE ONLY: tests,
 * the smoke check and the benchmark's CPU-baseline leg call it; the product
 * path never does.  It shares no code with the CUDA library.
 *
 * What it computes (chenxutan.com, "TileKernels 深度解析", section 4.1
 * "MoE Gating", the three-step naive form that the fused kernel replaces):
 *   1. logits = hidden_states @ gate_weight          (linear map, [T,H]x[H,E])
 *   2. topk_vals, topk_ids = topk(logits, k)          (k largest, in rank order)
 *   3. scores = softmax(topk_vals) over the k values
 *
 * Readings where the page is silent:
 *   - logits are exact-input fp64 sums (bf16 -> fp64 is exact, and each
 *     bf16 x bf16 product is exact in fp64); h runs 0..H-1 in order;
 *   - ranking is the strict total order (logit descending, expert index
 *     ascending), so equal logits go to the lower expert index; -0 == +0;
 *   - every row is fully sorted under that order and the first k are kept;
 *   - softmax is computed in fp64 as exp(v_j - v_0) / sum_i exp(v_i - v_0)
 *     (v_0 is the maximum), then rounded to fp32;
 *   - gap[t] = v_{k-1} - (the (k+1)-th largest logit), +inf when k == E.
 *
 * Parity pins: see tests/test_oracle_pins.py (brute-force subset enumeration,
 * a hand-worked example, closed forms, invariants, library cross-checks).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    double value;
    int32_t index;
} oracle_entry;

static double oracle_bf16_to_f64(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* qsort comparator for the total order: larger logit first, then lower index. */
static int oracle_rank_before(const void* pa, const void* pb) {
    const oracle_entry* a = (const oracle_entry*)pa;
    const oracle_entry* b = (const oracle_entry*)pb;
    if (a->value > b->value) return -1;
    if (a->value < b->value) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * hidden:   bf16 bits [T, H] row-major
 * gate:     bf16 bits [H, E] row-major
 * scores:   out fp32 [T, k]        scores64: out fp64 [T, k] (nullable)
 * ids:      out int32 [T, k]       gap:      out fp64 [T]    (nullable)
 * logits:   out fp64 [T, E] (nullable), the step-1 values
 * Returns 0 on success, -1 on a bad argument, -2 on allocation failure.
 */
int oracle_fused_topk_gating(const uint16_t* hidden, const uint16_t* gate, int64_t T, int64_t H, int64_t E,
                             int k, float* scores, double* scores64, int32_t* ids, double* gap,
                             double* logits) {
    if (T < 0 || H < 1 || E < 1 || k < 1 || k > E) return -1;
    if (T == 0) return 0;
    if (!hidden || !gate || !scores || !ids) return -1;

    /* gate widened to fp64 once (exact) */
    double* w = (double*)malloc(sizeof(double) * (size_t)(H * E));
    if (!w) return -2;
    for (int64_t i = 0; i < H * E; ++i) w[i] = oracle_bf16_to_f64(gate[i]);

    int failed = 0;
#pragma omp parallel
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)E);
        oracle_entry* row = (oracle_entry*)malloc(sizeof(oracle_entry) * (size_t)E);
        const int have_buffers = acc && row;
        if (!have_buffers) {
#pragma omp atomic write
            failed = 1;
        }
        {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < T; ++t) {
                if (!have_buffers) continue;
                const uint16_t* x = hidden + t * H;
                /* step 1: logits, summed over h in order for every expert */
                for (int64_t e = 0; e < E; ++e) acc[e] = 0.0;
                for (int64_t h = 0; h < H; ++h) {
                    const double xv = oracle_bf16_to_f64(x[h]);
                    const double* wr = w + h * E;
                    for (int64_t e = 0; e < E; ++e) acc[e] += xv * wr[e];
                }
                if (logits)
                    for (int64_t e = 0; e < E; ++e) logits[t * E + e] = acc[e];

                /* step 2: full sort under the total order, keep the first k */
                for (int64_t e = 0; e < E; ++e) {
                    row[e].value = acc[e] + 0.0; /* -0 -> +0 */
                    row[e].index = (int32_t)e;
                }
                qsort(row, (size_t)E, sizeof(oracle_entry), oracle_rank_before);

                /* step 3: softmax over the k selected values */
                const double m = row[0].value;
                double denom = 0.0;
                for (int j = 0; j < k; ++j) denom += exp(row[j].value - m);
                for (int j = 0; j < k; ++j) {
                    const double s = exp(row[j].value - m) / denom;
                    scores[t * k + j] = (float)s;
                    if (scores64) scores64[t * k + j] = s;
                    ids[t * k + j] = row[j].index;
                }
                if (gap) gap[t] = (k < E) ? row[k - 1].value - row[k].value : INFINITY;
            }
        }
        free(acc);
        free(row);
    }
    free(w);
    return failed ? -2 : 0;
}
