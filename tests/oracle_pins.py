"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` handle and raises
``AssertionError`` when the handle disagrees with what the definition (the
naive three-step gating form of chenxutan.com section 4.1) and plain
mathematics fix:

* brute force over every k-subset, with logits in exact rational arithmetic;
* a hand-worked two-token example (``golden/hand_worked_2token.json``);
* closed forms: k=2 scores are a logistic of the logit difference, a zero gate
  gives 1/k, k=1 is an argmax with the lowest index on ties;
* library routines for special cases: k=E is a stable descending argsort plus
  a full softmax (``scipy.special.softmax``); numpy's fp64 matmul (another
  summation order) agrees with the logits within rounding;
* invariants: distinct in-range ids, non-increasing scores summing to 1.

``tests/test_oracle_mutants.py`` plants plausible mistakes in copies of the
oracle source and checks that each one fails at least one pin.
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import scipy.special

import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits_from_values(values) -> np.ndarray:
    """bf16 bits of values that must be exactly representable in bf16."""
    v = np.asarray(values, dtype=np.float64)
    bits = workloads.round_bf16(v)
    assert np.array_equal(workloads.bf16_to_f64(bits), v), "value not exact in bf16"
    return bits


def _exact_logits(x_bits: np.ndarray, w_bits: np.ndarray) -> list:
    """Logits as exact rationals (bf16 values are dyadic, so this is exact)."""
    x = workloads.bf16_to_f64(x_bits)
    w = workloads.bf16_to_f64(w_bits)
    T, H = x.shape
    E = w.shape[1]
    xf = [[Fraction(float(v)) for v in row] for row in x]
    wf = [[Fraction(float(v)) for v in row] for row in w]
    return [[sum((xf[t][h] * wf[h][e] for h in range(H)), Fraction(0)) for e in range(E)] for t in range(T)]


def _brute_force_topk(row: list, k: int) -> list:
    """The unique k-subset S with key(s) before key(c) for every s in S, c not in S,
    where key = (logit descending, index ascending); returned in key order."""
    E = len(row)

    def before(a, b):
        return row[a] > row[b] or (row[a] == row[b] and a < b)

    found = []
    for subset in itertools.combinations(range(E), k):
        inside = set(subset)
        if all(before(s, c) for s in subset for c in range(E) if c not in inside):
            found.append(subset)
    assert len(found) == 1, f"total order must give one subset, got {len(found)}"
    chosen = list(found[0])
    # order inside the subset: insertion by the same key, pairwise
    ordered = []
    for s in chosen:
        pos = 0
        while pos < len(ordered) and before(ordered[pos], s):
            pos += 1
        ordered.insert(pos, s)
    return ordered


def _tiny_cases():
    """(x_bits, w_bits, k) tiny inputs: random normals and tie-heavy small integers."""
    cases = []
    rng_case = 0
    for (T, H, E, k) in [(48, 8, 12, 4), (40, 6, 16, 2), (32, 8, 10, 3), (24, 4, 7, 7), (24, 5, 9, 1)]:
        x = workloads.normal_bf16(100 + rng_case, 1, 0, T * H).reshape(T, H)
        w = workloads.normal_bf16(100 + rng_case, 2, 0, H * E, 1.0 / math.sqrt(H)).reshape(H, E)
        cases.append((x, w, k))
        rng_case += 1
    # small integers -> many exact ties between different experts
    for (T, H, E, k) in [(64, 3, 12, 4), (64, 2, 8, 3), (32, 4, 16, 5)]:
        ux = workloads.normal_f64(200 + rng_case, 1, 0, T * H)
        uw = workloads.normal_f64(200 + rng_case, 2, 0, H * E)
        x = _bits_from_values(np.clip(np.round(ux * 1.2), -3, 3).reshape(T, H))
        w = _bits_from_values(np.clip(np.round(uw * 1.2), -2, 2).reshape(H, E))
        cases.append((x, w, k))
        rng_case += 1
    return cases


# --------------------------------------------------------------------------
def pin_hand_worked(o) -> None:
    with open(os.path.join(GOLDEN, "hand_worked_2token.json")) as f:
        g = json.load(f)
    x = _bits_from_values(g["hidden"])
    w = _bits_from_values(g["gate_weight"])
    r = o.gating(x, w, g["k"], want_logits=True)
    exp = g["expected"]
    assert np.array_equal(r.logits, np.array(exp["logits"])), r.logits
    assert np.array_equal(r.ids, np.array(exp["ids"], dtype=np.int32)), r.ids
    s0 = 1.0 / (1.0 + math.exp(-0.5))
    s1 = math.exp(-0.5) / (1.0 + math.exp(-0.5))
    want = np.array([[s0, s1], [0.5, 0.5]])
    assert np.allclose(r.scores64, want, rtol=0, atol=1e-15), r.scores64
    assert np.array_equal(r.scores, want.astype(np.float32)), r.scores
    assert np.array_equal(r.gap, np.array(exp["gap"])), r.gap


def pin_brute_force(o) -> None:
    for x, w, k in _tiny_cases():
        exact = _exact_logits(x, w)
        r = o.gating(x, w, k, want_logits=True)
        for t, row in enumerate(exact):
            want = _brute_force_topk(row, k)
            assert r.ids[t].tolist() == want, (t, r.ids[t].tolist(), want)


def pin_exact_logits(o) -> None:
    for x, w, k in _tiny_cases():
        exact = _exact_logits(x, w)
        r = o.gating(x, w, k, want_logits=True)
        H = x.shape[1]
        xv, wv = workloads.bf16_to_f64(x), workloads.bf16_to_f64(w)
        for t, row in enumerate(exact):
            for e, val in enumerate(row):
                # each fp64 addition rounds once: |err| <= H * 2^-53 * sum |terms|
                bound = H * 2.0 ** -53 * float(np.sum(np.abs(xv[t] * wv[:, e])))
                assert abs(r.logits[t, e] - float(val)) <= bound, (t, e, r.logits[t, e], float(val))


def pin_numpy_matmul(o) -> None:
    wl = workloads.RouterWorkload("pin", 64, 512, 16, 4)
    x, w = wl.hidden(), wl.gate_weight()
    r = o.gating(x, w, wl.k, want_logits=True)
    ref = workloads.bf16_to_f64(x) @ workloads.bf16_to_f64(w)
    assert np.max(np.abs(r.logits - ref)) <= 1e-9


def pin_gap(o) -> None:
    for x, w, k in _tiny_cases():
        exact = _exact_logits(x, w)
        r = o.gating(x, w, k)
        E = w.shape[1]
        for t, row in enumerate(exact):
            ranked = sorted(row, reverse=True)
            want = math.inf if k == E else float(ranked[k - 1] - ranked[k])
            assert (r.gap[t] == want) if k == E else abs(r.gap[t] - want) <= 1e-12, (t, r.gap[t], want)


def pin_invariants(o) -> None:
    for wl in (workloads.RouterWorkload("inv", 200, 256, 64, 6),
               workloads.RouterWorkload("inv", 100, 96, 24, 24),
               workloads.RouterWorkload("inv", 50, 64, 16, 1)):
        r = o.gating(wl.hidden(), wl.gate_weight(), wl.k)
        assert np.all((r.ids >= 0) & (r.ids < wl.E))
        for row in r.ids:
            assert len(set(row.tolist())) == wl.k
        assert np.all(np.abs(r.scores.astype(np.float64).sum(axis=1) - 1.0) <= 1e-6)
        assert np.all(np.diff(r.scores64, axis=1) <= 0.0)
        assert np.all(r.scores64 > 0.0)


def pin_zero_gate(o) -> None:
    for (T, H, E, k) in [(16, 64, 16, 2), (8, 128, 64, 8), (4, 32, 16, 16)]:
        x = workloads.normal_bf16(7, 1, 0, T * H).reshape(T, H)
        w = np.zeros((H, E), dtype=np.uint16)
        r = o.gating(x, w, k)
        assert np.array_equal(r.ids, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
        assert np.all(np.abs(r.scores64 - 1.0 / k) <= 1e-15)
        assert np.all(np.abs(r.scores - np.float32(1.0 / k)) <= 1e-7)


def pin_k1_argmax(o) -> None:
    wl = workloads.RouterWorkload("k1", 300, 64, 32, 1)
    x, w = wl.hidden(), wl.gate_weight().copy()
    w[:, 9] = w[:, 3]    # exact duplicate columns: ties must go to the lower index
    w[:, 30] = w[:, 12]
    r = o.gating(x, w, 1, want_logits=True)
    ref = workloads.bf16_to_f64(x) @ workloads.bf16_to_f64(w)
    top2 = -np.sort(-ref, axis=1)[:, :2]
    d = top2[:, 0] - top2[:, 1]
    clear = (d == 0) | (d > 1e-9)  # numpy's summation order cannot flip these
    assert clear.sum() > 0.9 * wl.T
    assert np.array_equal(r.ids[clear, 0], np.argmax(ref, axis=1).astype(np.int32)[clear])
    assert np.all(r.scores == 1.0)


def pin_kE_full_softmax(o) -> None:
    for (T, H, E) in [(40, 64, 16), (20, 8, 24)]:
        wl = workloads.RouterWorkload("kE", T, H, E, E)
        x, w = wl.hidden(), wl.gate_weight().copy()
        w[:, E - 1] = w[:, 0]
        r = o.gating(x, w, E, want_logits=True)
        ref = workloads.bf16_to_f64(x) @ workloads.bf16_to_f64(w)
        order = np.argsort(-ref, axis=1, kind="stable")
        gaps = np.diff(np.take_along_axis(ref, order, axis=1), axis=1)
        # where numpy's summation order cannot flip a near-tie, the orders agree
        for t in range(T):
            if np.all((gaps[t] == 0) | (np.abs(gaps[t]) > 1e-9)):
                assert r.ids[t].tolist() == order[t].tolist(), (t, r.ids[t], order[t])
            want = scipy.special.softmax(ref[t][r.ids[t]])
            assert np.max(np.abs(r.scores64[t] - want)) <= 1e-12
        assert np.all(np.isinf(r.gap))


def pin_k2_logistic(o) -> None:
    wl = workloads.RouterWorkload("k2", 128, 256, 16, 2)
    r = o.gating(wl.hidden(), wl.gate_weight(), 2, want_logits=True)
    v = np.take_along_axis(r.logits, r.ids.astype(np.int64), axis=1)
    assert np.all(v[:, 0] >= v[:, 1])
    assert np.max(np.abs(r.scores64[:, 0] - scipy.special.expit(v[:, 0] - v[:, 1]))) <= 1e-15
    assert np.max(np.abs(r.scores64[:, 1] - scipy.special.expit(v[:, 1] - v[:, 0]))) <= 1e-15


ALL_PINS = [pin_hand_worked, pin_brute_force, pin_exact_logits, pin_numpy_matmul, pin_gap,
            pin_invariants, pin_zero_gate, pin_k1_argmax, pin_kE_full_softmax, pin_k2_logistic]
