"""Routing metadata on the GPU vs the CPU oracle (a stable counting sort),
bit-exact: offsets, sorted_slots and slot_pos are integers with one correct
answer (ascending assignment inside an expert), so every element must match.

Inputs are seeded expert ids (uniform and skewed popularity, k distinct per
row), ids the oracle's gating picked, and hand-made degenerate cases: no
assignment, one expert, every id equal, invalid ids, E not a multiple of 4,
the largest E, and sizes that leave ragged warp and CTA ranges.
"""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import workloads

pytestmark = pytest.mark.gpu

SENTINEL = -7  # written by neither side: marks elements the call must leave alone
GUARD = 64     # extra elements after each output, which must stay untouched


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0


def _guarded(n):
    return torch.full((n + GUARD,), SENTINEL, dtype=torch.int32, device="cuda")


def run_route(ids: np.ndarray, E: int, stream=None):
    """GPU route through the C ABI into guarded buffers; returns numpy results."""
    T, k = ids.shape
    n = T * k
    d_ids = torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).cuda()
    off, ss, sp = _guarded(E + 1), _guarded(n), _guarded(n)
    st = tk.route_ptr(d_ids.data_ptr(), T, k, E, off.data_ptr(), ss.data_ptr(), sp.data_ptr(),
                      0 if stream is None else stream.cuda_stream)
    assert st == tk.TK_OK, tk.status_string(st)
    torch.cuda.synchronize()
    off, ss, sp = off.cpu().numpy(), ss.cpu().numpy(), sp.cpu().numpy()
    for name, a, m in (("offsets", off, E + 1), ("sorted_slots", ss, n), ("slot_pos", sp, n)):
        assert (a[m:] == SENTINEL).all(), f"{name}: wrote past its end"
    return off[:E + 1], ss[:n], sp[:n]


def check(ids: np.ndarray, E: int, stream=None):
    off, ss, sp = run_route(ids, E, stream)
    ref = oracle.route(ids, E)
    placed = int(ref.offsets[E])
    assert np.array_equal(off, ref.offsets), "offsets differ"
    assert np.array_equal(sp, ref.slot_pos.reshape(-1)), "slot_pos differs"
    assert np.array_equal(ss[:placed], ref.sorted_slots[:placed]), "sorted_slots differ"
    assert (ss[placed:] == SENTINEL).all(), "positions past the placed count were written"
    return ref


@pytest.mark.parametrize("T,k,E,kind", [
    (1, 1, 16, "uniform"), (1, 8, 256, "uniform"), (512, 8, 256, "uniform"), (4097, 1, 16, "skew"),
    (513, 8, 256, "skew"), (7, 2, 16, "uniform"), (64, 2, 16, "uniform"),
    (37, 3, 5, "uniform"), (4096, 8, 256, "uniform"), (4096, 8, 256, "skew"), (16384, 6, 64, "skew"),
    (12345, 7, 999, "skew"), (3001, 16, 1024, "uniform"), (5000, 1, 1, "uniform"), (9999, 3, 13, "skew"),
    (65536, 8, 256, "uniform"), (65536, 8, 256, "skew"),
])
def test_route_matches_oracle(T, k, E, kind):
    check(workloads.expert_ids(T, k, E, seed=1000 + T + E, kind=kind), E)


def test_route_train_shape_ragged_ranges():
    # 65533 x 8 slots: the last warp range and the last CTA are partly filled
    T = 65533
    p = tk.route_plan(T, 8, 256)
    assert (T * 8) % p["warp_slots"] != 0 and p["ctas"] > 1
    check(workloads.expert_ids(T, 8, 256, seed=7, kind="skew"), 256)


def test_route_empty():
    off, _, _ = run_route(np.zeros((0, 8), dtype=np.int32), 256)
    assert (off == 0).all()


def test_route_every_id_equal():
    # whole warps fall in one match group; positions are plain ascending slots
    ids = np.full((20000, 4), 3, dtype=np.int32)
    ref = check(ids, 8)
    assert ref.offsets.tolist() == [0, 0, 0, 0] + [80000] * 5


def test_route_invalid_ids_are_not_placed():
    ids = workloads.expert_ids(5000, 8, 256, seed=11)
    rng = np.random.default_rng(12)
    flat = ids.reshape(-1)
    bad = rng.choice(flat.size, size=777, replace=False)
    flat[bad] = rng.choice(np.array([-1, 256, 257, 2**31 - 1, -2**31], dtype=np.int64), size=bad.size)
    ref = check(ids, 256)
    assert int(ref.offsets[256]) == flat.size - 777


def test_route_of_oracle_gating_ids():
    wl = workloads.TINY
    ids = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), wl.k).ids
    check(ids, wl.E)


def test_route_on_side_stream_and_repeated_calls():
    s = torch.cuda.Stream()
    for seed, (T, k, E) in enumerate([(4096, 8, 256), (100, 3, 7), (65536, 8, 256), (1, 1, 1)]):
        check(workloads.expert_ids(T, k, E, seed=seed), E, stream=s)


def check_route_properties(ids: np.ndarray, E: int, offsets, sorted_slots, slot_pos):
    """What any correct routing of ``ids`` satisfies (valid ids only), checked
    without the oracle: a permutation grouped by expert, ascending inside an
    expert, slot_pos its inverse, offsets the counts' exclusive prefix sum."""
    flat = ids.reshape(-1).astype(np.int64)
    n = flat.size
    assert ((flat >= 0) & (flat < E)).all()
    counts = np.bincount(flat, minlength=E)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(sorted_slots), np.arange(n))
    assert np.array_equal(slot_pos[sorted_slots], np.arange(n))
    e_sorted = flat[sorted_slots]
    assert (np.diff(e_sorted) >= 0).all()
    same = np.diff(e_sorted) == 0
    assert (np.diff(sorted_slots)[same] > 0).all()


def test_route_after_gating_on_device():
    # the chained use: gating ids stay on the device and feed routing directly;
    # the gating ids are checked by the gating parity tests, the routing of them
    # here by the properties any correct routing has
    wl = workloads.DEEPSEEK
    x = workloads.to_torch_bf16(wl.hidden()).cuda()
    w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
    _, ids = tk.fused_topk_gating(x, w, wl.k)
    offsets, sorted_slots, slot_pos = tk.route(ids, wl.E)
    torch.cuda.synchronize()
    check_route_properties(ids.cpu().numpy(), wl.E, offsets.cpu().numpy(), sorted_slots.cpu().numpy(),
                           slot_pos.cpu().numpy().reshape(-1))
