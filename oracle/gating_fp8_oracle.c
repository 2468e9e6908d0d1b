/*
 * CPU oracle for fused MoE top-k gating on FP8 (E4M3) inputs with scales.
 * TEST INFRASTRUCTURE ONLY (tests, the smoke check, the benchmark's CPU
 * baseline); it shares no code with the CUDA library.
 *
 * What it computes: the gating of chenxutan.com, "TileKernels 深度解析",
 * section 4.1 "MoE Gating" (logits, top-k, softmax over the k values) on
 * inputs quantized as in section 4.3 "Quantization" (FP8 E4M3 values with a
 * per-token scale, the page's per_token_quantize):
 *   hidden[t, h] = hidden_scale[t] * e4m3(hidden_q[t, h])
 *   gate[e, h]   = gate_scale[e]   * e4m3(gate_q[e, h])      (one scale per expert)
 *   logits[t, e] = sum_h hidden[t, h] * gate[e, h]           (fp64, h in order)
 * then the same total order, top-k and softmax as gating_oracle.c.  Readings
 * where the pages are silent: the gate is quantized too (a tensor-core FP8
 * product needs both operands in FP8), with one scale per expert, and stored
 * expert-major [E, H] (each expert's H values contiguous, with its scale).
 *
 * E4M3 ("FN": no infinities): sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; the
 * largest finite magnitude is 1.75 * 2^8 = 448.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double oracle_e4m3_to_f64(uint8_t bits) {
    const int sign = bits >> 7;
    const int exponent = (bits >> 3) & 0xF;
    const int mantissa = bits & 0x7;
    double magnitude;
    if (exponent == 0xF && mantissa == 0x7) return NAN;
    if (exponent == 0)
        magnitude = ldexp((double)mantissa / 8.0, -6);
    else
        magnitude = ldexp(1.0 + (double)mantissa / 8.0, exponent - 7);
    return sign ? -magnitude : magnitude;
}

typedef struct {
    double value;
    int32_t index;
} fp8_oracle_entry;

static int fp8_oracle_rank_before(const void* pa, const void* pb) {
    const fp8_oracle_entry* a = (const fp8_oracle_entry*)pa;
    const fp8_oracle_entry* b = (const fp8_oracle_entry*)pb;
    if (a->value > b->value) return -1;
    if (a->value < b->value) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

/*
 * hidden_q: e4m3 bits [T, H];  hidden_scale: [T]
 * gate_q:   e4m3 bits [E, H];  gate_scale:   [E]
 * outputs as oracle_fused_topk_gating (scores, scores64, ids, gap, logits).
 * Returns 0 on success, -1 on a bad argument, -2 on allocation failure.
 */
int oracle_fused_topk_gating_fp8(const uint8_t* hidden_q, const float* hidden_scale, const uint8_t* gate_q,
                                 const float* gate_scale, int64_t T, int64_t H, int64_t E, int k, float* scores,
                                 double* scores64, int32_t* ids, double* gap, double* logits) {
    if (T < 0 || H < 1 || E < 1 || k < 1 || k > E) return -1;
    if (T == 0) return 0;
    if (!hidden_q || !hidden_scale || !gate_q || !gate_scale || !scores || !ids) return -1;

    /* the dequantized gate, once */
    double* w = (double*)malloc(sizeof(double) * (size_t)(E * H));
    if (!w) return -2;
    for (int64_t e = 0; e < E; ++e)
        for (int64_t h = 0; h < H; ++h) w[e * H + h] = (double)gate_scale[e] * oracle_e4m3_to_f64(gate_q[e * H + h]);

    int failed = 0;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)H);
        fp8_oracle_entry* row = (fp8_oracle_entry*)malloc(sizeof(fp8_oracle_entry) * (size_t)E);
        const int have_buffers = x && row;
        if (!have_buffers) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < T; ++t) {
            if (!have_buffers) continue;
            for (int64_t h = 0; h < H; ++h) x[h] = (double)hidden_scale[t] * oracle_e4m3_to_f64(hidden_q[t * H + h]);
            for (int64_t e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int64_t h = 0; h < H; ++h) acc += x[h] * w[e * H + h];
                if (logits) logits[t * E + e] = acc;
                row[e].value = acc + 0.0; /* -0 -> +0 */
                row[e].index = (int32_t)e;
            }
            qsort(row, (size_t)E, sizeof(fp8_oracle_entry), fp8_oracle_rank_before);
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
        free(x);
        free(row);
    }
    free(w);
    return failed ? -2 : 0;
}
