"""Expert-parallel dispatch and combine: ``fused_dispatch`` / ``fused_combine``.

The two calls of the chenxutan.com page "TileKernels 深度解析", section 4.2
"MoE Routing": dispatch sends every token to the ranks that hold the experts
its ``expert_ids`` row names; combine brings the experts' results back and sums
them weighted by the gating scores.  In a group of R ranks, rank q holds
experts [q * E / R, (q + 1) * E / R) and receives, for each of them in
ascending order, each source rank's rows for it (sources ascending, each in
ascending assignment order t * k + j).

Every step on the data runs in the library's kernels: the routing metadata
(``tk_gating_route``), the row-address tables (``tk_gating_ep_rows_table``),
the copy of each token row straight into its destination buffer
(``tk_gating_fused_dispatch``) and the weighted gather-sum that pulls the
expert outputs from where they lie (``tk_gating_fused_combine``).  This module
marshals arguments and runs the small control exchange: each rank's
per-expert counts, gathered over the process group, and, once per group,
the inter-process handles of every rank's buffers.

With one rank everything stays on the caller's stream, except one read of the
routing offsets (to size the returned view and check every rank's capacity).  With several, ranks
order their steps with process-group barriers after synchronising their
stream (each rank's dispatch must be complete before any expert reads a
receive buffer, and every expert output before any combine reads it).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

from . import _binding as _b

IPC_HANDLE_BYTES = 128


def _lib():
    lib = _b.library()
    if not getattr(lib, "_ep_bound", False):
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        lib.tk_gating_fused_dispatch.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp]
        lib.tk_gating_fused_dispatch.restype = ctypes.c_int
        lib.tk_gating_fused_combine.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.tk_gating_fused_combine.restype = ctypes.c_int
        lib.tk_gating_ep_rows_table.argtypes = [vp, i32, i32, i32, vp, vp, i64, vp, vp, vp, vp]
        lib.tk_gating_ep_rows_table.restype = ctypes.c_int
        lib.tk_gating_ep_ipc_handle.argtypes = [vp, vp]
        lib.tk_gating_ep_ipc_handle.restype = ctypes.c_int
        lib.tk_gating_ep_ipc_open.argtypes = [vp, ctypes.POINTER(ctypes.c_void_p)]
        lib.tk_gating_ep_ipc_open.restype = ctypes.c_int
        lib.tk_gating_ep_ipc_close.argtypes = [vp, vp]
        lib.tk_gating_ep_ipc_close.restype = ctypes.c_int
        lib._ep_bound = True
    return lib


# ---------------------------------------------------------------------------
# host logic: the layout of the receive buffers (also used to size them)
# ---------------------------------------------------------------------------
@dataclass
class ExchangePlan:
    """Layout of one exchange, from every rank's per-expert counts."""
    R: int
    E: int
    rank: int
    recv_rows: list          # rows each rank receives
    recv_offsets: list       # per rank q: its experts' first rows in its buffer (length E/R + 1)
    dest_row: list           # for `rank` as source: the first row of its block of expert e


def received_rows(offsets_all, R: int, E: int) -> list:
    """Rows each rank receives, from every rank's routing offsets ([R][E + 1])."""
    per = E // R
    rows = [0] * R
    for s in range(R):
        o = offsets_all[s]
        for q in range(R):
            rows[q] += int(o[(q + 1) * per]) - int(o[q * per])
    return rows


def check_capacities(offsets_all, capacities) -> list:
    """The rows each rank receives; ValueError when one exceeds its capacity.
    Every rank runs this on the same gathered offsets, so all of them refuse
    together and no rank writes past another's buffer."""
    R = len(capacities)
    E = len(offsets_all[0]) - 1
    rows = received_rows(offsets_all, R, E)
    over = [q for q in range(R) if rows[q] > capacities[q]]
    if over:
        q = over[0]
        raise ValueError(f"rank {q} would receive {rows[q]} rows; its capacity is {capacities[q]}")
    return rows


def exchange_plan(counts, rank: int) -> ExchangePlan:
    """``counts[s][e]``: assignments of source rank s to expert e (R x E)."""
    R = len(counts)
    E = len(counts[0]) if R else 0
    if R < 1 or E % R != 0:
        raise ValueError(f"{E} experts do not split over {R} ranks")
    per = E // R
    total = [sum(int(counts[s][e]) for s in range(R)) for e in range(E)]
    recv_offsets, recv_rows = [], []
    for q in range(R):
        offs = [0]
        for e in range(q * per, (q + 1) * per):
            offs.append(offs[-1] + total[e])
        recv_offsets.append(offs)
        recv_rows.append(offs[-1])
    dest_row = []
    for e in range(E):
        q = e // per
        dest_row.append(recv_offsets[q][e - q * per] + sum(int(counts[s][e]) for s in range(rank)))
    return ExchangePlan(R, E, rank, recv_rows, recv_offsets, dest_row)


# ---------------------------------------------------------------------------
def _check(st: int, where: str) -> None:
    if st != _b.TK_OK:
        raise _b.TkGatingError(st, where)


def _stream(stream, device) -> int:
    import torch
    return int((stream or torch.cuda.current_stream(device)).cuda_stream)


def dispatch_rows(tokens, ids, offsets, slot_pos, rows, num_experts: int, stream=None) -> None:
    """Raw dispatch with a row-address table ``rows`` (uint64 [E] on the device);
    ``offsets`` and ``slot_pos`` are tk_gating_route's for ``ids``."""
    T, H = tokens.shape
    k = ids.shape[1]
    with _device(tokens):
        _check(_lib().tk_gating_fused_dispatch(tokens.data_ptr(), T, H, k, int(num_experts), ids.data_ptr(),
                                               offsets.data_ptr(), slot_pos.data_ptr(), rows.data_ptr(),
                                               _stream(stream, tokens.device)), "tk_gating_fused_dispatch")


def combine_rows(rows, ids, offsets, slot_pos, scores, out, num_experts: int, stream=None) -> None:
    """Raw combine with a row-address table ``rows`` (uint64 [E] on the device)."""
    T, H = out.shape
    k = ids.shape[1]
    with _device(out):
        _check(_lib().tk_gating_fused_combine(rows.data_ptr(), T, H, k, int(num_experts), ids.data_ptr(),
                                              offsets.data_ptr(), slot_pos.data_ptr(), scores.data_ptr(),
                                              out.data_ptr(), _stream(stream, out.device)), "tk_gating_fused_combine")


def rows_table(offsets_all, rank: int, bases, out_bases, H: int, stream=None):
    """(rows, out_rows, recv_offsets) device tables from every rank's routing
    offsets, int32 [R, E + 1] on the device, and uint64 base-address tensors [R]
    (see tk_gating_ep_rows_table)."""
    import torch
    R, E1 = offsets_all.shape
    E = E1 - 1
    dev = offsets_all.device
    rows = torch.empty(E, dtype=torch.uint64, device=dev)
    out_rows = torch.empty(E, dtype=torch.uint64, device=dev) if out_bases is not None else None
    recv_offsets = torch.empty(E // R + 1, dtype=torch.int32, device=dev)
    with _device(offsets_all):
        _check(_lib().tk_gating_ep_rows_table(
            offsets_all.data_ptr(), R, E, int(rank), bases.data_ptr(),
            out_bases.data_ptr() if out_bases is not None else None, int(H), rows.data_ptr(),
            out_rows.data_ptr() if out_rows is not None else None, recv_offsets.data_ptr(), _stream(stream, dev)),
            "tk_gating_ep_rows_table")
    return rows, out_rows, recv_offsets


class _device:
    def __init__(self, t):
        import torch
        self._ctx = torch.cuda.device(t.device)

    def __enter__(self):
        self._ctx.__enter__()

    def __exit__(self, *exc):
        self._ctx.__exit__(*exc)


def ipc_handle(tensor) -> bytes:
    """The inter-process handle of a CUDA tensor's memory (TK_EP_IPC_HANDLE_BYTES bytes)."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    with _device(tensor):
        _check(_lib().tk_gating_ep_ipc_handle(tensor.data_ptr(), buf), "tk_gating_ep_ipc_handle")
    return buf.raw


def ipc_open(handle: bytes) -> int:
    """The address, in this process, of the buffer another process exported."""
    p = ctypes.c_void_p(0)
    _check(_lib().tk_gating_ep_ipc_open(handle, ctypes.byref(p)), "tk_gating_ep_ipc_open")
    return int(p.value)


def ipc_close(address: int, handle: bytes) -> None:
    _check(_lib().tk_gating_ep_ipc_close(address, handle), "tk_gating_ep_ipc_close")


# ---------------------------------------------------------------------------
@dataclass
class DispatchHandle:
    """What combine needs from dispatch (the page's dispatch_indices)."""
    ids: object           # int32 [T, k]
    offsets: object       # int32 [E + 1]
    slot_pos: object      # int32 [T, k]
    out_rows: object      # uint64 [E]: where each expert's output rows for this rank lie
    recv_offsets: object  # int32 [E/R + 1]: this rank's experts in its receive buffer (device)
    recv_rows: int        # rows this rank received


class ExpertParallelGroup:
    """The buffers of one rank of an expert-parallel group.

    Every rank allocates a receive buffer and an expert-output buffer of
    ``capacity`` rows of ``hidden`` bf16 values; with several ranks their
    inter-process handles are exchanged once over ``group`` and opened, so each
    rank holds every rank's buffer addresses.  ``group`` is a torch.distributed
    process group (None: the default group, or a single rank when
    torch.distributed is not initialised); its collectives carry only the
    counts, the handles and barriers.
    """

    def __init__(self, num_experts: int, hidden: int, capacity: int, group=None, device=None):
        import torch
        import torch.distributed as dist
        self.E, self.H, self.capacity = int(num_experts), int(hidden), int(capacity)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.group = group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.R = dist.get_world_size(group) if self.distributed else 1
        self.rank = dist.get_rank(group) if self.distributed else 0
        if self.E % self.R != 0:
            raise ValueError(f"{self.E} experts do not split over {self.R} ranks")
        self.recv = torch.empty((self.capacity, self.H), dtype=torch.bfloat16, device=self.device)
        self.output = torch.empty((self.capacity, self.H), dtype=torch.bfloat16, device=self.device)
        self._opened = []
        if self.R == 1:
            bases = [self.recv.data_ptr()]
            out_bases = [self.output.data_ptr()]
            self.capacities = [self.capacity]
        else:
            mine = (ipc_handle(self.recv), ipc_handle(self.output), self.capacity)
            allh = [None] * self.R
            dist.all_gather_object(allh, mine, group=group)
            bases, out_bases = [], []
            self.capacities = [int(c) for (_, _, c) in allh]
            with torch.cuda.device(self.device):
                for q, (hr, ho, _) in enumerate(allh):
                    if q == self.rank:
                        bases.append(self.recv.data_ptr())
                        out_bases.append(self.output.data_ptr())
                    else:
                        a, b = ipc_open(hr), ipc_open(ho)
                        self._opened += [(a, hr), (b, ho)]
                        bases.append(a)
                        out_bases.append(b)
        self.bases = torch.tensor(bases, dtype=torch.uint64, device=self.device)
        self.out_bases = torch.tensor(out_bases, dtype=torch.uint64, device=self.device)

    def close(self) -> None:
        for a, h in self._opened:
            ipc_close(a, h)
        self._opened = []

    # -- control plane ------------------------------------------------------
    def _barrier(self, stream=None) -> None:
        import torch
        import torch.distributed as dist
        if self.R > 1:
            (stream or torch.cuda.current_stream(self.device)).synchronize()
            dist.barrier(group=self.group)

    def _gather_offsets(self, offsets):
        """Every rank's routing offsets, int32 [R, E + 1] on this device."""
        import torch
        import torch.distributed as dist
        if self.R == 1:
            return offsets.view(1, self.E + 1)
        if dist.get_backend(self.group) == "nccl":
            out = torch.empty((self.R, self.E + 1), dtype=torch.int32, device=self.device)
            dist.all_gather_into_tensor(out, offsets, group=self.group)
            return out
        host = [torch.empty(self.E + 1, dtype=torch.int32) for _ in range(self.R)]
        dist.all_gather(host, offsets.cpu(), group=self.group)
        return torch.stack(host).to(self.device)

    # -- the two calls ---------------------------------------------------------
    def fused_dispatch(self, tokens, expert_ids, stream=None):
        """Send every row of ``tokens`` [T, H] bf16 to the experts ``expert_ids``
        [T, k] int32 names.  Returns (this rank's received rows [N, H] -- a view
        of the receive buffer --, the handle combine needs).  Write the experts'
        outputs, row for row, into ``self.output[:N]`` before combine."""
        import torch
        from . import _binding as b
        if tokens.shape[1] != self.H or tokens.dtype != torch.bfloat16:
            raise ValueError(f"tokens must be bf16 [T, {self.H}]")
        offsets, sorted_slots, slot_pos = b.route(expert_ids, self.E, stream=stream)
        offsets_all = self._gather_offsets(offsets)
        # every rank checks every destination (the same numbers on all ranks): the
        # dispatch below writes into other ranks' buffers
        recv_rows = check_capacities(offsets_all.cpu().tolist(), self.capacities)[self.rank]
        rows, out_rows, recv_offsets = rows_table(offsets_all, self.rank, self.bases, self.out_bases, self.H, stream)
        self._barrier(stream)  # every receive buffer is free
        dispatch_rows(tokens, expert_ids, offsets, slot_pos, rows, self.E, stream)
        self._barrier(stream)  # every rank's rows have landed
        return self.recv[:recv_rows], DispatchHandle(expert_ids, offsets, slot_pos, out_rows, recv_offsets, recv_rows)

    def fused_combine(self, handle: DispatchHandle, scores, out=None, stream=None):
        """``out[t] = sum_j scores[t, j] * (expert output of assignment (t, j))``,
        pulled from every rank's output buffer; bf16 [T, H]."""
        import torch
        T, k = handle.ids.shape
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        self._barrier(stream)  # every expert output is written
        combine_rows(handle.out_rows, handle.ids, handle.offsets, handle.slot_pos, scores, out, self.E, stream)
        self._barrier(stream)  # nobody overwrites an output buffer still being read
        return out
