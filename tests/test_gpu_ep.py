"""Expert-parallel dispatch and combine on the GPU against the oracle.

* One rank: ``ExpertParallelGroup`` end to end (routing, row table, dispatch
  into the receive buffer, experts applied by the test, pull-mode combine).
* Several ranks emulated in one process on one GPU: each rank's receive and
  output buffers are separate allocations; every source rank's dispatch
  launch writes into all of them through its row table and every rank's
  combine reads from all of them -- the kernels and tables a multi-GPU group
  uses, with local instead of peer addresses.  The launches do not wait on
  one another; the test orders them on one stream.
* Two processes on the one GPU: the receive and output buffers of each are
  opened in the other through the inter-process handles, and the ranks order
  their steps with gloo barriers (host side), as a multi-GPU group does.

Dispatch is a copy, compared bit for bit.  Combine sums k products in fp32
(fused multiply-adds in rank order) and rounds once to bf16; the oracle sums
in fp64.  Tolerance: half a bf16 unit in the last place of the exact value
(the final rounding) plus k * 2^-24 * sum_j |s_j y_j| (the fp32 roundings).
"""
import os
import socket

import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import workloads
from moe_router_gating_b200 import ep
from oracle import ep_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0, "an expert-parallel kernel reported a bad row address"


def bf16_bits_to_torch(bits):
    return workloads.to_torch_bf16(bits)


def expert_scale(E):
    """The test's experts: expert e multiplies its rows by c_e (exact in bf16)."""
    return np.array([0.5 + (e % 7) * 0.25 for e in range(E)], dtype=np.float64)


def apply_experts(rows_bits, experts_of_rows, c):
    """bf16 bits of c_e * row (rounded to bf16 like any expert output)."""
    vals = ep_oracle.bf16_to_f64(rows_bits) * c[experts_of_rows][:, None]
    return workloads.round_bf16(vals)


def check_combine(got_bits, want_f64, terms_abs, k):
    got = ep_oracle.bf16_to_f64(got_bits)
    mag = np.maximum(np.abs(want_f64), np.abs(got))  # the rounded sum may sit one binade up
    exp = np.floor(np.log2(np.maximum(mag, 1e-300)))
    half_ulp = np.where(mag != 0, 2.0 ** (exp - 8), 0.0)
    bound = half_ulp + k * 2.0 ** -24 * terms_abs + 1e-30
    err = np.abs(got - want_f64)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"combine off at {bad[0]}: {got[tuple(bad[0])]} vs {want_f64[tuple(bad[0])]}"


def run_case(R, T, H, k, E, seed, kind="uniform"):
    """Emulated ranks on one GPU: tokens, ids, scores per rank; returns nothing, asserts."""
    dev = torch.device("cuda")
    toks = [workloads.normal_bf16(seed + s, 1, 0, T[s] * H).reshape(T[s], H) for s in range(R)]
    ids = [workloads.expert_ids(T[s], k, E, seed=seed + 50 + s, kind=kind) for s in range(R)]
    rng = np.random.default_rng(seed)
    scores = [rng.random((T[s], k)).astype(np.float32) for s in range(R)]
    want = ep_oracle.dispatch(toks, ids, E)
    cap = max(1, max(len(r) for r in want.rows))
    recv = [torch.full((cap, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16) for _ in range(R)]
    outb = [torch.zeros((cap, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    bases = torch.tensor([r.data_ptr() for r in recv], dtype=torch.uint64, device=dev)
    out_bases = torch.tensor([o.data_ptr() for o in outb], dtype=torch.uint64, device=dev)
    d_ids = [torch.from_numpy(i).to(dev) for i in ids]
    routes = [tk.route(d, E) for d in d_ids]
    offsets_all = torch.stack([r[0] for r in routes])
    tables = [ep.rows_table(offsets_all, s, bases, out_bases, H) for s in range(R)]
    # the device tables against the host plan of the same counts
    counts = np.diff(offsets_all.cpu().numpy().astype(np.int64), axis=1)
    base_list = bases.cpu().numpy().astype(np.uint64)
    out_list = out_bases.cpu().numpy().astype(np.uint64)
    for s in range(R):
        plan = ep.exchange_plan(counts, s)
        per = E // R
        rows = tables[s][0].cpu().numpy().astype(np.uint64)
        orows = tables[s][1].cpu().numpy().astype(np.uint64)
        for e in range(E):
            q = e // per
            assert int(rows[e]) == int(base_list[q]) + plan.dest_row[e] * 2 * H, (s, e)
            assert int(orows[e]) == int(out_list[q]) + plan.dest_row[e] * 2 * H, (s, e)
    for s in range(R):  # every source rank's dispatch writes into every receive buffer
        x = bf16_bits_to_torch(toks[s]).to(dev)
        ep.dispatch_rows(x, d_ids[s], routes[s][0], routes[s][2], tables[s][0], E)
    torch.cuda.synchronize()
    per = E // R
    for q in range(R):
        n = len(want.rows[q])
        got = recv[q][:n].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, want.rows[q]), f"receive buffer of rank {q}"
        assert np.array_equal(tables[q][2].cpu().numpy(), np.concatenate([[0], np.cumsum(want.expert_counts[q])]))
        # the test's experts, on the received rows (experts of rows from the oracle's counts)
        experts_of_rows = np.repeat(np.arange(q * per, (q + 1) * per), want.expert_counts[q])
        y = apply_experts(want.rows[q], experts_of_rows, expert_scale(E))
        outb[q][:n].copy_(bf16_bits_to_torch(y).to(dev))
    torch.cuda.synchronize()
    ys = [ep_oracle.bf16_to_f64(outb[q][:len(want.rows[q])].view(torch.int16).cpu().numpy().view(np.uint16))
          for q in range(R)]
    want_out = ep_oracle.combine(ys, want, scores, list(T))
    abs_terms = ep_oracle.combine([np.abs(y) for y in ys], want, [np.abs(sc) for sc in scores], list(T))
    for s in range(R):
        out = torch.empty((T[s], H), dtype=torch.bfloat16, device=dev)
        sc = torch.from_numpy(scores[s]).to(dev)
        ep.combine_rows(tables[s][1], d_ids[s], routes[s][0], routes[s][2], sc, out, E)
        torch.cuda.synchronize()
        check_combine(out.view(torch.int16).cpu().numpy().view(np.uint16), want_out[s], abs_terms[s], k)


@pytest.mark.parametrize("R,T,H,k,E,kind", [
    (1, (300,), 256, 8, 64, "uniform"),
    (1, (4096,), 7168, 8, 256, "skew"),
    (2, (257, 300), 512, 4, 16, "skew"),
    (4, (100, 1, 0, 333), 128, 3, 32, "uniform"),
    (8, (64,) * 8, 7168, 8, 256, "uniform"),
    (2, (2000, 1500), 1024, 32, 64, "skew"),
    (1, (513,), 3592, 8, 64, "uniform"),   # combine rows in three parts, the last one shorter
])
def test_emulated_ranks_match_the_oracle(R, T, H, k, E, kind):
    run_case(R, T, H, k, E, seed=R * 7 + k, kind=kind)


def test_group_api_one_rank():
    T, H, k, E = 1000, 1024, 8, 64
    dev = torch.device("cuda")
    toks = workloads.normal_bf16(3, 1, 0, T * H).reshape(T, H)
    ids = workloads.expert_ids(T, k, E, seed=9, kind="skew")
    scores = np.random.default_rng(2).random((T, k)).astype(np.float32)
    g = ep.ExpertParallelGroup(E, H, capacity=T * k, device=dev)
    recv, handle = g.fused_dispatch(bf16_bits_to_torch(toks).to(dev), torch.from_numpy(ids).to(dev))
    want = ep_oracle.dispatch([toks], [ids], E)
    assert handle.recv_rows == len(want.rows[0])
    assert np.array_equal(recv.view(torch.int16).cpu().numpy().view(np.uint16), want.rows[0])
    experts_of_rows = np.repeat(np.arange(E), want.expert_counts[0])
    y = apply_experts(want.rows[0], experts_of_rows, expert_scale(E))
    g.output[:handle.recv_rows].copy_(bf16_bits_to_torch(y).to(dev))
    out = g.fused_combine(handle, torch.from_numpy(scores).to(dev))
    torch.cuda.synchronize()
    yf = [ep_oracle.bf16_to_f64(y)]
    want_out = ep_oracle.combine(yf, want, [scores], [T])[0]
    abs_terms = ep_oracle.combine([np.abs(yf[0])], want, [np.abs(scores)], [T])[0]
    check_combine(out.view(torch.int16).cpu().numpy().view(np.uint16), want_out, abs_terms, k)


def test_misaligned_row_address_is_reported_not_written():
    T, H, k, E = 16, 64, 2, 16
    dev = torch.device("cuda")
    x = torch.ones((T, H), dtype=torch.bfloat16, device=dev)
    ids = torch.from_numpy(workloads.expert_ids(T, k, E, seed=1)).to(dev)
    offsets, sorted_slots, slot_pos = tk.route(ids, E)
    buf = torch.zeros(T * k * H + 64, dtype=torch.bfloat16, device=dev)
    rows = torch.tensor([buf.data_ptr() + 2] * E, dtype=torch.uint64, device=dev)  # 2 bytes off alignment
    tk.device_error(clear=True)
    ep.dispatch_rows(x, ids, offsets, slot_pos, rows, E)
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) & (1 << 8)
    assert torch.count_nonzero(buf) == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        T, H, k, E = 400 + 37 * rank, 512, 4, 16
        toks = workloads.normal_bf16(rank, 1, 0, T * H).reshape(T, H)
        ids = workloads.expert_ids(T, k, E, seed=30 + rank, kind="skew")
        scores = np.random.default_rng(rank).random((T, k)).astype(np.float32)
        g = ep.ExpertParallelGroup(E, H, capacity=(400 + 37) * k * world, device=dev)
        recv, handle = g.fused_dispatch(bf16_bits_to_torch(toks).to(dev), torch.from_numpy(ids).to(dev))
        got = recv.view(torch.int16).cpu().numpy().view(np.uint16).copy()
        # the experts: c_e * row, experts of this rank's rows from its receive offsets
        offs = handle.recv_offsets.cpu().numpy()
        per = E // world
        experts_of_rows = np.repeat(np.arange(rank * per, (rank + 1) * per), np.diff(offs))
        y = apply_experts(got, experts_of_rows, expert_scale(E))
        g.output[:handle.recv_rows].copy_(bf16_bits_to_torch(y).to(dev))
        out = g.fused_combine(handle, torch.from_numpy(scores).to(dev))
        torch.cuda.synchronize()
        q.put((rank, got, y, out.view(torch.int16).cpu().numpy().view(np.uint16)))
        g.close()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_processes_share_buffers_through_ipc_handles():
    import multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, rows, y, out = q.get(timeout=300)
        got[r] = (rows, y, out)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    T = [400 + 37 * r for r in range(world)]
    H, k, E = 512, 4, 16
    toks = [workloads.normal_bf16(r, 1, 0, T[r] * H).reshape(T[r], H) for r in range(world)]
    ids = [workloads.expert_ids(T[r], k, E, seed=30 + r, kind="skew") for r in range(world)]
    scores = [np.random.default_rng(r).random((T[r], k)).astype(np.float32) for r in range(world)]
    want = ep_oracle.dispatch(toks, ids, E)
    for r in range(world):
        assert np.array_equal(got[r][0], want.rows[r]), f"receive buffer of rank {r}"
    ys = [ep_oracle.bf16_to_f64(got[r][1]) for r in range(world)]
    want_out = ep_oracle.combine(ys, want, scores, T)
    abs_terms = ep_oracle.combine([np.abs(y) for y in ys], want, [np.abs(s) for s in scores], T)
    for r in range(world):
        check_combine(got[r][2], want_out[r], abs_terms[r], k)
