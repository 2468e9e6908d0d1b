"""CPU oracle for expert-parallel dispatch and combine -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module; the product never does, and it imports nothing from
the product.

What it computes (chenxutan.com, "TileKernels 深度解析", section 4.2 "MoE
Routing": ``fused_dispatch(tokens, expert_ids, num_experts, ep_group)`` sends
each token to the GPUs of the experts its expert_ids row names and returns the
indices ``fused_combine(expert_output, dispatch_indices, scores, ep_group)``
uses to bring the experts' results back, weighted by the gating scores):

* an expert-parallel group of R ranks; rank q holds experts
  [q * E / R, (q + 1) * E / R);
* dispatch: rank q receives, for each of its experts e in ascending order,
  for each source rank s in ascending order, the token rows of s's
  assignments (t, j) with ids_s[t, j] == e, in ascending t * k + j;
* combine: source rank s gets out_s[t] = sum_j scores_s[t, j] * y[(t, j)],
  where y[(t, j)] is the expert output row at the place dispatch put the
  assignment (t, j).  Assignments whose id is outside [0, E) take no part.

The readings (receive order, ascending assignment order inside an expert and
source, the scores summed in fp64 here) are this library's; the page shows
only the two calls.  Plain Python loops over the definition; numpy only for
bf16 widening and the fp64 sums.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclass
class Dispatched:
    rows: list            # per destination rank q: uint16 bf16 bits [N_q, H]
    expert_counts: list   # per destination rank q: int64 [E / R] rows per local expert
    where: list           # per source rank s: dict (t, j) -> (q, row) for every valid assignment


def dispatch(tokens: list, ids: list, E: int) -> Dispatched:
    """``tokens[s]``: bf16 bits [T_s, H]; ``ids[s]``: int32 [T_s, k]; R = len(tokens)."""
    R = len(tokens)
    if E % R != 0:
        raise ValueError("the experts must split evenly over the ranks")
    per = E // R
    H = tokens[0].shape[1]
    # the assignments of each (expert, source rank), in ascending t * k + j
    bucket = {}
    for s in range(R):
        T_s, k = ids[s].shape
        for t in range(T_s):
            for j in range(k):
                e = int(ids[s][t, j])
                if 0 <= e < E:
                    bucket.setdefault((e, s), []).append((t, j))
    rows, counts = [], []
    where = [dict() for _ in range(R)]
    for q in range(R):
        out = []
        cnt = np.zeros(per, dtype=np.int64)
        for e in range(q * per, (q + 1) * per):      # the destination's experts, ascending
            for s in range(R):                        # then the source ranks, ascending
                for (t, j) in bucket.get((e, s), []):
                    where[s][(t, j)] = (q, len(out))
                    out.append(tokens[s][t])
                    cnt[e - q * per] += 1
        rows.append(np.array(out, dtype=np.uint16).reshape(len(out), H))
        counts.append(cnt)
    return Dispatched(rows, counts, where)


def combine(expert_out: list, dispatched: Dispatched, scores: list, T: list) -> list:
    """``expert_out[q]``: float64 [N_q, H] (the experts' rows in rank q's receive
    order); returns per source rank s the float64 [T_s, H] weighted sums."""
    R = len(expert_out)
    H = expert_out[0].shape[1] if expert_out and expert_out[0].ndim == 2 else 0
    outs = []
    for s in range(R):
        k = scores[s].shape[1] if scores[s].ndim == 2 else 0
        o = np.zeros((T[s], H), dtype=np.float64)
        for t in range(T[s]):
            for j in range(k):
                loc = dispatched.where[s].get((t, j))
                if loc is not None:
                    q, r = loc
                    o[t] += float(scores[s][t, j]) * expert_out[q][r]
        outs.append(o)
    return outs
