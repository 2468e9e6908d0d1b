"""Pins of the expert-parallel dispatch/combine oracle (CPU only).

Each pin reaches the oracle's result by another route: the independently
pinned routing oracle (one rank), a library sort of all assignments by
(expert, source rank, assignment), and closed forms of combine.  Planted
mistakes in copies of the oracle must each fail a pin."""
import inspect
import sys
import types

import numpy as np
import pytest

import oracle
import workloads
from oracle import ep_oracle


def _ranks(R, T, H, k, E, seed, kind="uniform", invalid=0):
    toks, ids = [], []
    for s in range(R):
        toks.append(workloads.normal_bf16(seed + s, 1, 0, T[s] * H).reshape(T[s], H))
        i = workloads.expert_ids(T[s], k, E, seed=seed + 100 + s, kind=kind)
        if invalid and T[s]:
            i = i.copy()
            i.reshape(-1)[:: max(1, i.size // invalid)] = E + 3   # ids outside [0, E) take no part
        ids.append(i)
    return toks, ids


def _lexsort_layout(ids, E, R):
    """(q, source, t, j) of every receive row, by a library sort of (expert, source, slot)."""
    recs = []
    for s, i in enumerate(ids):
        T_s, k = i.shape
        for t in range(T_s):
            for j in range(k):
                e = int(i[t, j])
                if 0 <= e < E:
                    recs.append((e, s, t * k + j, t, j))
    recs = np.array(recs, dtype=np.int64).reshape(-1, 5)
    order = np.lexsort((recs[:, 2], recs[:, 1], recs[:, 0])) if len(recs) else np.zeros(0, np.int64)
    per = E // R
    layout = [[] for _ in range(R)]
    for r in recs[order]:
        layout[int(r[0]) // per].append((int(r[1]), int(r[3]), int(r[4])))
    return layout


def check_pins(mod, R=3, T=(37, 0, 64), H=16, k=3, E=12, seed=4, invalid=5):
    toks, ids = _ranks(R, list(T), H, k, E, seed, invalid=invalid)
    d = mod.dispatch(toks, ids, E)
    # layout from a library sort of (expert, source rank, assignment)
    layout = _lexsort_layout(ids, E, R)
    for q in range(R):
        assert d.rows[q].shape == (len(layout[q]), H)
        for r, (s, t, j) in enumerate(layout[q]):
            assert np.array_equal(d.rows[q][r], toks[s][t]), (q, r)
            assert d.where[s][(t, j)] == (q, r)
        per = E // R
        want = np.bincount([int(ids[s][t, j]) - q * per for (s, t, j) in layout[q]], minlength=per)
        assert np.array_equal(d.expert_counts[q], want)
    # combine, closed form with scaled experts: y = c_e * row  =>  out[t] = x_t * sum_j s_j c_{e_j}
    c = np.linspace(0.5, 2.0, E)
    expert_out = []
    for q in range(R):
        ys = np.zeros((len(layout[q]), H))
        for r, (s, t, j) in enumerate(layout[q]):
            ys[r] = c[int(ids[s][t, j])] * ep_oracle.bf16_to_f64(toks[s][t])
        expert_out.append(ys)
    rng = np.random.default_rng(seed)
    scores = [rng.random((T[s], k)).astype(np.float32) for s in range(R)]
    outs = mod.combine(expert_out, d, scores, list(T))
    for s in range(R):
        valid = (ids[s] >= 0) & (ids[s] < E)
        w = np.where(valid, scores[s].astype(np.float64) * c[np.clip(ids[s], 0, E - 1)], 0.0).sum(axis=1)
        want = ep_oracle.bf16_to_f64(toks[s]) * w[:, None]
        assert np.allclose(outs[s], want, rtol=1e-12, atol=1e-12), s


def test_pins_hold():
    check_pins(ep_oracle)
    check_pins(ep_oracle, R=2, T=(50, 41), k=4, E=8, invalid=0, seed=9)
    check_pins(ep_oracle, R=4, T=(20, 31, 7, 12), k=2, E=16, invalid=3, seed=2)


def test_one_rank_equals_the_routing_oracle():
    T, H, k, E = 300, 8, 4, 32
    toks, ids = _ranks(1, [T], H, k, E, seed=5, kind="skew")
    d = ep_oracle.dispatch(toks, ids, E)
    r = oracle.route(ids[0], E)
    assert np.array_equal(d.rows[0], toks[0][r.sorted_slots // k])
    for t in range(T):
        for j in range(k):
            assert d.where[0][(t, j)] == (0, int(r.slot_pos[t * k + j]))
    assert np.array_equal(np.concatenate([[0], np.cumsum(d.expert_counts[0])]), r.offsets)


def test_identity_experts_with_uniform_scores_return_the_tokens():
    T, H, k, E = 40, 8, 4, 8
    toks, ids = _ranks(2, [T, T], H, k, E, seed=6)
    d = ep_oracle.dispatch(toks, ids, E)
    outs = ep_oracle.combine([ep_oracle.bf16_to_f64(r) for r in d.rows], d,
                             [np.full((T, k), 1.0 / k, np.float32)] * 2, [T, T])
    for s in range(2):
        assert np.array_equal(outs[s], ep_oracle.bf16_to_f64(toks[s]))  # 1/4 sums exactly


def _mutant(old: str, new: str):
    src = inspect.getsource(ep_oracle)
    assert old in src, old
    mod = types.ModuleType("ep_mutant")
    sys.modules["ep_mutant"] = mod  # dataclasses look their module up
    try:
        exec(compile(src.replace(old, new, 1), "ep_mutant", "exec"), mod.__dict__)
    finally:
        del sys.modules["ep_mutant"]
    return mod


@pytest.mark.parametrize("old,new", [
    ("for s in range(R):                        # then", "for s in reversed(range(R)):              # then"),
    ("for e in range(q * per, (q + 1) * per):", "for e in reversed(range(q * per, (q + 1) * per)):"),
    ("if 0 <= e < E:", "if 0 <= e < E and (t + j) % 17 != 5:"),
    ("o[t] += float(scores[s][t, j]) * expert_out[q][r]", "o[t] += float(scores[s][t, (j + 1) % k]) * expert_out[q][r]"),
    ("out.append(tokens[s][t])", "out.append(tokens[s][min(t + 1, len(tokens[s]) - 1)])"),
    ("                e = int(ids[s][t, j])\n                if 0 <= e < E:",
     "                e = int(ids[s][t, j]) % E\n                if 0 <= e < E:"),   # invalid ids placed
])
def test_planted_mistakes_fail_a_pin(old, new):
    with pytest.raises((AssertionError, IndexError, KeyError)):
        check_pins(_mutant(old, new))
