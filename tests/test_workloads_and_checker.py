"""Input generator properties and the parity checker itself (CPU only)."""
import numpy as np
import pytest

import oracle
import parity
import workloads


def test_generator_is_counter_based():
    whole = workloads.normal_bf16(0, 1, 0, 10_001)
    part = workloads.normal_bf16(0, 1, 4_321, 777)
    assert np.array_equal(whole[4_321:4_321 + 777], part)
    assert not np.array_equal(workloads.normal_bf16(0, 2, 0, 1000), whole[:1000])
    assert not np.array_equal(workloads.normal_bf16(1, 1, 0, 1000), whole[:1000])


def test_generator_moments():
    z = workloads.normal_f64(0, 1, 0, 400_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1.0) < 0.01
    # Box-Muller pairs: cos and sin halves are uncorrelated
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 0.01


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, -0.0, 1e-3])
    got = workloads.bf16_to_f64(workloads.round_bf16(vals))
    assert got[0] == 1.0
    assert got[1] == 1.0                       # tie -> even
    assert got[2] == 1.0 + 4 * 2 ** -8          # tie -> even (up)
    assert got[3] == -2.5
    assert abs(got[6] - 1e-3) <= 1e-3 * 2 ** -8


def test_rows_match_whole_tensor():
    wl = workloads.RouterWorkload("t", 37, 40, 16, 2)
    assert np.array_equal(wl.hidden()[11:20], wl.hidden_rows(11, 9))
    sk = workloads.SKEW.with_T(9)
    assert np.array_equal(sk.hidden()[3:7], sk.hidden_rows(3, 4))


def test_skew_structure():
    sk = workloads.SKEW.with_T(64)
    w = sk.gate_weight()
    for a, b in sk.duplicate_pairs:
        assert np.array_equal(w[:, a], w[:, b])
    for d in sk.dominant:
        assert np.array_equal(w[:, d], w[:, sk.dominant[0]])
    u = sk.unit_vector()
    assert abs(np.dot(u, u) - 1.0) < 1e-12
    # the dominant experts (identical columns, logit ~ 3 + N(0,1)) win on most tokens
    r = oracle.fused_topk_gating(sk.hidden(), w, sk.k, want_logits=True)
    hits = np.isin(r.ids[:, :4], np.array(sk.dominant)).mean()
    assert hits > 0.75


def test_algorithmic_work():
    assert workloads.TRAIN.algorithmic_bytes() == 947_388_416
    assert workloads.DEEPSEEK.algorithmic_bytes() == 62_652_416
    assert workloads.SKEW.algorithmic_bytes() == 135_528_448
    assert workloads.TRAIN.flops() == 2 * 65536 * 7168 * 256


# ---- the checker: accepts the oracle's own answer, rejects planted errors ----
@pytest.fixture(scope="module")
def case():
    wl = workloads.RouterWorkload("chk", 256, 128, 32, 4)
    x, w = wl.hidden(), wl.gate_weight().copy()
    w[:, 21] = w[:, 20]
    r = oracle.fused_topk_gating(x, w, wl.k, want_logits=True)
    return r


def test_checker_accepts_oracle(case):
    parity.check(case.scores, case.ids, case, duplicate_pairs=((20, 21),))


def test_checker_rejects_wrong_set(case):
    ids = case.ids.copy()
    t = int(np.argmax(case.gap))
    ids[t, -1] = next(e for e in range(32) if e not in ids[t])
    with pytest.raises(AssertionError):
        parity.check(case.scores, ids, case)


def test_checker_rejects_score_error(case):
    sc = case.scores.copy()
    sc[3, 0] += 2e-3
    with pytest.raises(AssertionError):
        parity.check(sc, case.ids, case)


def test_checker_rejects_far_swap(case):
    ids = case.ids.copy()
    ol = np.take_along_axis(case.logits, case.ids.astype(np.int64), axis=1)
    t = int(np.argmax(ol[:, 0] - ol[:, 1]))
    ids[t, 0], ids[t, 1] = ids[t, 1], ids[t, 0]
    with pytest.raises(AssertionError):
        parity.check(case.scores, ids, case)


def test_checker_rejects_duplicate_order(case):
    rows = np.nonzero(np.any(case.ids == 20, axis=1) & np.any(case.ids == 21, axis=1))[0]
    assert rows.size > 0
    ids = case.ids.copy()
    t = rows[0]
    pa, pb = int(np.nonzero(ids[t] == 20)[0][0]), int(np.nonzero(ids[t] == 21)[0][0])
    ids[t, pa], ids[t, pb] = 21, 20
    with pytest.raises(AssertionError):
        parity.check(case.scores, ids, case, duplicate_pairs=((20, 21),))


def test_own_selection_checker_accepts_the_rule_and_rejects_mistakes():
    # ties resolve to the lower index, -0.0 equals +0.0
    L = np.array([[0.5, 2.0, 2.0, -1.0, 0.0, -0.0],
                  [-0.0, 0.0, -3.0, -0.0, 1.0, 1.0]], dtype=np.float32)
    ids = np.array([[1, 2, 0, 4], [4, 5, 0, 1]], dtype=np.int32)
    v = np.take_along_axis(L, ids, axis=1).astype(np.float64)
    s = np.exp(v - v[:, :1]) / np.exp(v - v[:, :1]).sum(axis=1, keepdims=True)
    assert parity.check_own_selection(s.astype(np.float32), ids, L) == 2
    swapped = ids.copy()
    swapped[0, :2] = [2, 1]                        # equal values in the wrong index order
    with pytest.raises(AssertionError):
        parity.check_own_selection(s.astype(np.float32), swapped, L)
    zero_order = ids.copy()
    zero_order[1, 2:] = [1, 0]                     # -0.0 and +0.0 are equal: index order decides
    with pytest.raises(AssertionError):
        parity.check_own_selection(s.astype(np.float32), zero_order, L)
    with pytest.raises(AssertionError):            # a wrong score
        parity.check_own_selection((s + 1e-4).astype(np.float32), ids, L)


def test_logit_error_is_the_largest_difference():
    a = np.zeros((3, 4))
    b = a.copy()
    b[2, 1] = -3e-5
    assert parity.logit_error(b.astype(np.float32), a) == pytest.approx(3e-5, rel=1e-3)
