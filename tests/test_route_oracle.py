"""Pins for the routing oracle (CPU): numpy's stable argsort and bincount are
independent library routines for the same definition; invariants cover the
rest (a permutation, grouped by expert, ascending inside an expert)."""
import numpy as np
import pytest

import oracle

ROUTE_MUTANTS = {
    "descending_slots": ("for (int64_t s = 0; s < n; ++s) {\n        const int32_t e = ids[s];",
                         "for (int64_t s = n - 1; s >= 0; --s) {\n        const int32_t e = ids[s];"),
    "inclusive_offsets": ("        offsets[e] = (int32_t)run;\n        next[e] = run;\n        run += count[e];",
                          "        run += count[e];\n        offsets[e] = (int32_t)run;\n        next[e] = run - count[e];"),
    "position_off_by_one": ("const int64_t p = next[e]++;", "const int64_t p = ++next[e] - (e == 0);"),
    "wrong_inverse": ("slot_pos[s] = (int32_t)p;", "slot_pos[s] = (int32_t)(p ^ (p & 1));"),
}


def _ids(T, k, E, seed, skew=False):
    rng = np.random.default_rng(seed)
    if skew:
        p = rng.dirichlet(np.full(E, 0.3))
        return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


CASES = [(1, 1, 16, False), (7, 2, 16, False), (300, 8, 256, False), (1000, 6, 64, True), (513, 16, 256, True)]


def _pin_library_routines(o, T, k, E, skew):
    ids = _ids(T, k, E, seed=T + E, skew=skew)
    r = o.route(ids, E)
    flat = ids.reshape(-1)
    assert np.array_equal(r.sorted_slots, np.argsort(flat, kind="stable").astype(np.int32))
    counts = np.bincount(flat, minlength=E)
    assert np.array_equal(r.offsets, np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
    assert np.array_equal(r.slot_pos[r.sorted_slots], np.arange(flat.size))


@pytest.mark.parametrize("T,k,E,skew", CASES)
def test_matches_stable_argsort_and_bincount(T, k, E, skew):
    _pin_library_routines(oracle.load(), T, k, E, skew)


@pytest.mark.parametrize("name", sorted(ROUTE_MUTANTS))
def test_route_mutant_is_caught(name, tmp_path):
    before, after = ROUTE_MUTANTS[name]
    src = open(oracle.ROUTE_SOURCE).read()
    assert src.count(before) == 1, name
    mutant_src = tmp_path / "route_mutant.c"
    mutant_src.write_text(src.replace(before, after))
    mutant = oracle.Oracle(oracle.compile_oracle(oracle.SOURCE, str(tmp_path / "libm.so"), str(mutant_src)))
    caught = False
    for case in CASES:
        try:
            _pin_library_routines(mutant, *case)
        except AssertionError:
            caught = True
            break
    assert caught, f"route mutant {name} passed every pin"


def test_invariants_and_degenerate_cases():
    E = 32
    ids = np.full((50, 4), 0, dtype=np.int32)  # every assignment to one expert... (duplicates allowed here)
    ids[:, 1:] = [5, 9, 31]
    r = oracle.route(ids, E)
    assert r.offsets[0] == 0 and r.offsets[E] == ids.size
    assert np.all(np.diff(r.offsets) >= 0)
    flat = ids.reshape(-1)
    # grouped by expert, ascending slot inside an expert
    assert np.all(np.diff(flat[r.sorted_slots]) >= 0)
    for e in (0, 5, 9, 31):
        run = r.sorted_slots[r.offsets[e]:r.offsets[e + 1]]
        assert np.all(np.diff(run) > 0) and np.all(flat[run] == e)
    # empty input
    r0 = oracle.route(np.zeros((0, 8), dtype=np.int32), 16)
    assert np.array_equal(r0.offsets, np.zeros(17, dtype=np.int32))


def test_out_of_range_ids_are_left_out():
    ids = np.array([[0, 3], [-1, 2], [7, 3]], dtype=np.int32)  # E = 4: -1 and 7 are out of range
    r = oracle.route(ids, 4)
    assert r.slot_pos[2] == -1 and r.slot_pos[4] == -1
    assert r.offsets.tolist() == [0, 1, 1, 2, 4]
    assert r.sorted_slots[:4].tolist() == [0, 3, 1, 5]
