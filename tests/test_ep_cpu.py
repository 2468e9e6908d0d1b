"""Expert-parallel exchange, host side (CPU only): the receive-buffer layout
(``ep.exchange_plan``) against the oracle's definition, and the control
protocol of several ranks -- every rank's routing offsets gathered over a
process group, each rank's rows placed by the plan -- run as world-size-2
gloo ranks.  The copies themselves run in CUDA kernels on a GPU; here each
rank moves its rows with plain array indexing following the plan, which is
exactly what the kernels do with the table the plan describes."""
import os
import socket

import numpy as np
import pytest

import oracle
import workloads
from moe_router_gating_b200 import ep
from oracle import ep_oracle


def _counts(ids, E):
    out = np.zeros(E, dtype=np.int64)
    for e in ids.reshape(-1):
        if 0 <= e < E:
            out[e] += 1
    return out


def _place(plan, tokens, ids, E, recv):
    """Rank plan.rank's rows into the receive buffers, by the plan and its own routing."""
    r = oracle.route(ids, E)
    k = ids.shape[1]
    per = E // plan.R
    for p in range(int(r.offsets[E])):
        s = int(r.sorted_slots[p])
        e = int(ids.reshape(-1)[s])
        recv[e // per][plan.dest_row[e] + p - int(r.offsets[e])] = tokens[s // k]
    return r


@pytest.mark.parametrize("R,E,T,k", [(1, 16, 50, 4), (2, 8, 37, 3), (4, 16, 20, 2), (3, 12, 64, 5)])
def test_plan_places_every_row_where_the_oracle_does(R, E, T, k):
    H = 8
    toks = [workloads.normal_bf16(s, 1, 0, T * H).reshape(T, H) for s in range(R)]
    ids = [workloads.expert_ids(T, k, E, seed=10 + s, kind="skew") for s in range(R)]
    want = ep_oracle.dispatch(toks, ids, E)
    counts = [_counts(i, E) for i in ids]
    recv = None
    for s in range(R):
        plan = ep.exchange_plan(counts, s)
        if recv is None:
            assert plan.recv_rows == [len(x) for x in want.rows]
            for q in range(R):
                assert plan.recv_offsets[q] == [0] + list(np.cumsum(want.expert_counts[q]))
            recv = [np.zeros((n, H), dtype=np.uint16) for n in plan.recv_rows]
        _place(plan, toks[s], ids[s], E, recv)
    for q in range(R):
        assert np.array_equal(recv[q], want.rows[q])


def test_plan_rejects_uneven_expert_split():
    with pytest.raises(ValueError):
        ep.exchange_plan([[1, 2, 3], [0, 0, 0]], 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, E, T, k, H, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        toks = workloads.normal_bf16(rank, 1, 0, T * H).reshape(T, H)
        ids = workloads.expert_ids(T, k, E, seed=20 + rank, kind="skew")
        offsets = torch.from_numpy(oracle.route(ids, E).offsets.astype(np.int32))
        # the control exchange the product runs: every rank's routing offsets
        gathered = [torch.empty(E + 1, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, offsets)
        counts = [np.diff(g.numpy()) for g in gathered]
        plan = ep.exchange_plan(counts, rank)
        # every rank places its rows into the (shared, here gathered) receive buffers
        recv = [np.zeros((n, H), dtype=np.uint16) for n in plan.recv_rows]
        _place(plan, toks, ids, E, recv)
        mine = [torch.from_numpy(r.astype(np.int32)) for r in recv]
        summed = []
        for qq in range(world):  # a rank's buffer is the sum of what every source placed (disjoint rows)
            t = mine[qq].clone()
            dist.all_reduce(t)
            summed.append(t.numpy().astype(np.uint16))
        q.put((rank, summed[rank]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_offsets_and_place_rows():
    import multiprocessing as mp
    world, E, T, k, H = 2, 8, 33, 3, 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, E, T, k, H, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    toks = [workloads.normal_bf16(r, 1, 0, T * H).reshape(T, H) for r in range(world)]
    ids = [workloads.expert_ids(T, k, E, seed=20 + r, kind="skew") for r in range(world)]
    want = ep_oracle.dispatch(toks, ids, E)
    for r in range(world):
        assert np.array_equal(got[r], want.rows[r]), r


def test_capacity_check_sees_every_destination():
    # two ranks, four experts: rank 0 holds experts 0-1, rank 1 experts 2-3
    offsets_all = [[0, 3, 5, 9, 10],    # rank 0's routing: counts 3, 2, 4, 1
                   [0, 1, 1, 6, 8]]     # rank 1's routing: counts 1, 0, 5, 2
    assert ep.received_rows(offsets_all, 2, 4) == [3 + 2 + 1 + 0, 4 + 1 + 5 + 2]
    assert ep.check_capacities(offsets_all, [6, 12]) == [6, 12]
    with pytest.raises(ValueError, match="rank 1"):
        ep.check_capacities(offsets_all, [100, 11])   # another rank's buffer would overflow
    with pytest.raises(ValueError, match="rank 0"):
        ep.check_capacities(offsets_all, [5, 100])
