/*
 * CPU oracle for the local routing metadata of MoE dispatch.  TEST
 * INFRASTRUCTURE ONLY (tests, the benchmark's CPU-baseline leg); it shares no
 * code with the CUDA library.
 *
 * What it computes (chenxutan.com, "TileKernels 深度解析", section 4.2 "MoE
 * Routing": dispatch sends each token to the experts `expert_ids[num_tokens,
 * top_k]` names and returns the indices that combine uses to put results
 * back): for the n = T * k assignments s = t * k + j (token t, rank j) with
 * expert ids[s], the assignments grouped by expert.  Reading taken where the
 * page is silent: inside an expert, assignments keep ascending s (a stable
 * order, so the result is unique).
 *
 *   offsets[e]      = number of assignments to experts < e   (offsets[E] = n)
 *   sorted_slots[p] = the assignment at position p of the expert-grouped order
 *   slot_pos[s]     = the position of assignment s (the inverse permutation)
 *
 * This is a counting sort, written out: count, exclusive prefix sum, then
 * place the assignments in ascending s.  Ids outside [0, E) are not placed:
 * their slot_pos is -1 and they are left out of the counts.
 */
#include <stdint.h>
#include <stdlib.h>

int oracle_route(const int32_t* ids, int64_t n, int32_t E, int32_t* offsets, int32_t* sorted_slots,
                 int32_t* slot_pos) {
    if (n < 0 || E < 1 || !offsets || (n > 0 && (!ids || !sorted_slots || !slot_pos))) return -1;
    int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    int64_t* next = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!count || !next) {
        free(count);
        free(next);
        return -2;
    }
    for (int64_t s = 0; s < n; ++s)
        if (ids[s] >= 0 && ids[s] < E) count[ids[s]] += 1;
    int64_t run = 0;
    for (int32_t e = 0; e < E; ++e) {
        offsets[e] = (int32_t)run;
        next[e] = run;
        run += count[e];
    }
    offsets[E] = (int32_t)run;
    for (int64_t s = 0; s < n; ++s) {
        const int32_t e = ids[s];
        if (e < 0 || e >= E) {
            slot_pos[s] = -1;
            continue;
        }
        const int64_t p = next[e]++;
        sorted_slots[p] = (int32_t)s;
        slot_pos[s] = (int32_t)p;
    }
    free(count);
    free(next);
    return 0;
}
