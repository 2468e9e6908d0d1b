"""Parity rule between the CUDA path and the CPU oracle (same seeded inputs).

The oracle ranks fp64 logits; the kernel ranks fp32 tensor-core logits.  Where
two logits are closer than fp32 rounding the two may order them differently, so
the comparison follows the tolerance that the operator's specification states:

1. ids are distinct and inside ``[0, E)`` on every row;
2. where the oracle gap between the k-th and (k+1)-th logit exceeds ``GAP``,
   the id set equals the oracle's, and the order equals the oracle's except
   between adjacent ranks whose oracle logits differ by at most ``GAP``;
3. otherwise every selected id has oracle logit >= (oracle k-th logit - GAP);
4. ``|score_gpu - score_oracle| <= SCORE_ATOL`` at every rank;
5. scores are non-increasing along each row;
6. for duplicated gate columns (a < b, exactly equal logits), b is never
   selected without a, and a comes before b.
"""
from __future__ import annotations

import numpy as np

GAP = 2e-3
SCORE_ATOL = 1e-3


def check(gpu_scores: np.ndarray, gpu_ids: np.ndarray, oracle_result, rows=None,
          duplicate_pairs=(), label: str = "") -> dict:
    """Raise AssertionError on the first violated rule; return summary counts.

    ``oracle_result`` must carry fp64 ``logits``.  ``rows`` maps each oracle row
    to the GPU row it was computed for (default: identity).
    """
    o = oracle_result
    assert o.logits is not None, "parity needs the oracle's fp64 logits"
    T, k = o.ids.shape
    E = o.logits.shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    g_ids = np.asarray(gpu_ids)[rows].astype(np.int64)
    g_sc = np.asarray(gpu_scores)[rows].astype(np.float64)
    assert g_ids.shape == (T, k) and g_sc.shape == (T, k), (g_ids.shape, (T, k))

    # rule 1
    assert np.all((g_ids >= 0) & (g_ids < E)), f"{label}: id out of range"
    srt = np.sort(g_ids, axis=1)
    assert np.all(srt[:, 1:] != srt[:, :-1]) if k > 1 else True, f"{label}: repeated id in a row"

    wide = o.gap > GAP
    o_ids = o.ids.astype(np.int64)
    # rule 2: sets
    same_set = np.all(np.sort(o_ids, axis=1) == srt, axis=1)
    bad = np.nonzero(wide & ~same_set)[0]
    assert bad.size == 0, (f"{label}: id set differs on wide-gap row {rows[bad[0]]}: gpu {g_ids[bad[0]]} "
                           f"oracle {o_ids[bad[0]]} gap {o.gap[bad[0]]}")
    # rule 2: order, allowing swaps between near-equal adjacent ranks
    ol = np.take_along_axis(o.logits, o_ids, axis=1)
    swaps = 0
    for t in np.nonzero(wide)[0]:
        if np.array_equal(g_ids[t], o_ids[t]):
            continue
        j = 0
        while j < k:
            # a run of ranks whose consecutive oracle logits are within GAP may be permuted
            r = j
            while r + 1 < k and ol[t, r] - ol[t, r + 1] <= GAP:
                r += 1
            assert set(g_ids[t, j:r + 1].tolist()) == set(o_ids[t, j:r + 1].tolist()), (
                f"{label}: order differs beyond near-ties on row {rows[t]}: gpu {g_ids[t]} oracle {o_ids[t]}")
            j = r + 1
        swaps += 1
    # rule 3
    tau = ol[:, k - 1]
    g_logit = np.take_along_axis(o.logits, g_ids, axis=1)
    narrow = ~wide
    if narrow.any():
        worst = np.min(g_logit[narrow] - tau[narrow, None])
        assert worst >= -GAP, f"{label}: a narrow-gap row picked a logit {worst} below the k-th"
    # rule 4
    err = np.max(np.abs(g_sc - o.scores64)) if T else 0.0
    assert err <= SCORE_ATOL, f"{label}: score error {err}"
    # rule 5
    if k > 1:
        assert np.all(np.diff(g_sc, axis=1) <= 0.0), f"{label}: scores increase along a row"
    # rule 6
    for a, b in duplicate_pairs:
        has_a = np.any(g_ids == a, axis=1)
        has_b = np.any(g_ids == b, axis=1)
        assert not np.any(has_b & ~has_a), f"{label}: expert {b} chosen without its duplicate {a}"
        both = np.nonzero(has_a & has_b)[0]
        for t in both:
            pa = int(np.nonzero(g_ids[t] == a)[0][0])
            pb = int(np.nonzero(g_ids[t] == b)[0][0])
            assert pa < pb, f"{label}: duplicate {b} ranked before {a} on row {rows[t]}"
    return {"rows": int(T), "wide_gap_rows": int(wide.sum()), "reordered_rows": swaps,
            "max_score_err": float(err)}


# The kernels' fp32 logits against the oracle's fp64 logits.  A logit sums
# H = 7168 exact bf16 products in H / 16 = 448 fp32 tensor-core steps (FP8:
# 224); each step rounds a running sum of magnitude <~ 4 at relative 2^-24,
# about 2.4e-7.  Modelled as a random walk of those roundings the error has
# sigma ~ sqrt(448) * 2.4e-7 / 2 ~ 2.5e-6; the largest of tens of millions of
# logits lies several sigma out.  Measured on B200 (every logit of each
# workload): at most 5.4e-5 (65536 x 7168 x 1024), 5.0e-5 (65536 x 7168 x 256),
# 9.4e-6 (4096 x 7168 x 256), 1.4e-6 (one token); FP8 inputs at most 6.6e-6.
# The bound is 20x under GAP, the selection tolerance above, which therefore
# never hides a logit error.
LOGIT_ATOL = 1e-4
# softmax of the kernel's own fp32 values: fp32 expf, sum and division
OWN_SCORE_ATOL = 2e-6


def logit_error(gpu_logits: np.ndarray, oracle_logits: np.ndarray) -> float:
    """Largest |logit_gpu - logit_oracle| over every token and expert."""
    g = np.asarray(gpu_logits, dtype=np.float64)
    assert g.shape == oracle_logits.shape, (g.shape, oracle_logits.shape)
    return float(np.max(np.abs(g - oracle_logits))) if g.size else 0.0


def check_own_selection(gpu_scores: np.ndarray, gpu_ids: np.ndarray, gpu_logits: np.ndarray, label: str = "") -> int:
    """The selection and softmax the kernel made from its own fp32 logits, exactly.

    ids must be the first k of the (value descending, index ascending) order of
    the row's fp32 logits -- a stable sort of the negated values, in which -0.0
    and +0.0 compare equal -- and scores the softmax of those k values
    (computed here in fp64) within OWN_SCORE_ATOL.  Returns the row count.
    """
    L = np.asarray(gpu_logits, dtype=np.float32)
    ids = np.asarray(gpu_ids).astype(np.int64)
    T, k = ids.shape
    order = np.argsort(-L, axis=1, kind="stable")[:, :k]
    bad = np.nonzero(np.any(order != ids, axis=1))[0]
    assert bad.size == 0, (f"{label}: row {bad[0]} ids {ids[bad[0]]} are not the top-{k} of its own logits "
                           f"{order[bad[0]]}")
    v = np.take_along_axis(L, ids, axis=1).astype(np.float64)
    e = np.exp(v - v[:, :1])
    s = e / e.sum(axis=1, keepdims=True)
    err = float(np.max(np.abs(s - np.asarray(gpu_scores, dtype=np.float64)))) if T else 0.0
    assert err <= OWN_SCORE_ATOL, f"{label}: scores differ from the softmax of the selected logits by {err}"
    return T
