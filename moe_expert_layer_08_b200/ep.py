"""Expert parallelism across ranks, one process per GPU: the dispatch, expert
layer and combine of "Mega moe fusion with symmetric memory" (Procedure,
step 5) with the cross-rank exchange as all-to-all-v collectives of
torch.distributed (NCCL over NVLink between GPUs).

Rank r of R holds experts [r E/R, (r+1) E/R) in the packet layout.  A step
on each rank:

1. ``dispatch``: the library's routing packs the rank's routed rows (FP8 row,
   UE8M0 scales, local expert id), grouped by destination rank, and counts
   them per rank;
2. the counts (all_gather), then the rows (all_to_all_single) cross ranks;
3. ``expert``: the expert layer over the received rows with E/R experts, k = 1
   and weight 1, whose output is each row's bf16 expert output Y unchanged;
4. the outputs go back (the reverse all_to_all_single);
5. ``combine``: the library's top-k-weighted sum through the inverse
   permutation of step 1.

Every step of the computation runs in the CUDA library; this module sizes the
buffers and issues the collectives.

``forward_peers`` is the same step over peer memory: the ranks' receive and
output buffers are mapped into every rank's address space once
(``enable_peers``: CUDA IPC handles exchanged over the process group, see
``PeerBuffers``), the dispatch writes each routed row straight into the
receive buffers of the rank that holds its expert (``moe_ep_dispatch_peers``)
and the combine reads each expert output where it was computed
(``moe_ep_combine_peers``), with stream-ordered barriers (an all-reduce of one
element on the step's stream) between the phases instead of the row
all-to-alls.  Every rank takes the same collective
steps in the same order, whatever its row counts.  The row counts are needed
on the host for the split sizes, so ``forward`` synchronises once per step
after the count exchange (an all-gather of every rank's per-destination
counts).
"""
from __future__ import annotations

import torch

from . import (check_device_error, ep_combine, ep_combine_peers, ep_dispatch, ep_dispatch_peers, ep_route,
               ep_workspace_bytes, forward, ipc_close, ipc_handle, ipc_open, workspace_bytes)

__all__ = ["ExpertParallelLayer", "PeerBuffers", "CudaIpc"]


class CudaIpc:
    """The library's CUDA IPC entry points (moe_ipc_handle / _open / _close)."""

    def export(self, t):
        return ipc_handle(t)

    def open(self, handle: bytes, device: int) -> int:
        return ipc_open(handle, device)

    def close(self, base: int) -> None:
        ipc_close(base)


class PeerBuffers:
    """Named buffers of every rank of ``group``, addressable from this process.

    Every rank passes its own buffers (same names on every rank); each is
    exported as (IPC handle of its allocation, byte offset in it), the records
    are all-gathered, and every other rank's allocation is opened once (two
    buffers in one allocation share a handle).  ``tables[name]`` is an i64
    [ranks] tensor on ``device``: entry d is the address of rank d's buffer in
    this process (this rank's own buffer's address for d = rank).  A
    collective: every rank of the group constructs it at the same point.
    ``ipc`` is the mapping backend (default: CUDA IPC through the library).
    """

    def __init__(self, buffers: dict, group=None, ipc=None, device=None):
        import torch.distributed as dist
        self.ipc = ipc if ipc is not None else CudaIpc()
        self.rank, self.ranks = dist.get_rank(group), dist.get_world_size(group)
        names = sorted(buffers)
        first = buffers[names[0]]
        dev_index = first.device.index if first.device.type == "cuda" else -1
        mine = {n: self.ipc.export(buffers[n]) for n in names}
        everyone = [None] * self.ranks
        dist.all_gather_object(everyone, {"device": dev_index, "names": names, "records": mine}, group=group)
        if any(r["names"] != names for r in everyone):
            raise ValueError("every rank must pass the same buffer names")
        self.opened = {}  # handle bytes -> mapped base
        addr = {n: [0] * self.ranks for n in names}
        for d in range(self.ranks):
            for n in names:
                if d == self.rank:
                    addr[n][d] = buffers[n].data_ptr()
                    continue
                handle, offset = everyone[d]["records"][n]
                if handle not in self.opened:
                    self.opened[handle] = self.ipc.open(handle, dev_index)
                addr[n][d] = self.opened[handle] + offset
        dev = device if device is not None else first.device
        self.tables = {n: torch.tensor(addr[n], dtype=torch.int64, device=dev) for n in names}

    def close(self):
        """Unmaps the other ranks' allocations (after every kernel that uses them)."""
        for base in self.opened.values():
            self.ipc.close(base)
        self.opened = {}


class ExpertParallelLayer:
    """One rank's share of an expert-parallel MoE layer.

    l1_t, l2_t: the packet buffers (``transform_weights``) of this rank's E/R
    experts; E, k, H, I: the layer's sizes (E counts all ranks' experts);
    T_max: tokens per step on this rank; recv_max: rows this rank can receive
    per step (default R * T_max * k, every slot of every rank); rank, ranks:
    this rank and the rank count (default: from the initialised default
    process group, else 0 and 1); group: the process group of the exchange.
    """

    def __init__(self, l1_t, l2_t, E: int, k: int, H: int, I: int, T_max: int, recv_max: int | None = None,
                 rank: int | None = None, ranks: int | None = None, group=None, device=None):
        import torch.distributed as dist
        live = dist.is_available() and dist.is_initialized()
        self.group = group
        self.ranks = ranks if ranks is not None else (dist.get_world_size(group) if live else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if live else 0)
        if E % self.ranks != 0:
            raise ValueError(f"E = {E} is not a multiple of the rank count {self.ranks}")
        if not 0 <= self.rank < self.ranks:
            raise ValueError("rank out of range")
        self.l1_t, self.l2_t = l1_t, l2_t
        self.E, self.k, self.H, self.I, self.T_max = E, k, H, I, T_max
        self.E_loc = E // self.ranks
        self.recv_max = recv_max if recv_max is not None else self.ranks * T_max * k
        dev = torch.device(device) if device is not None else (l1_t.device if l1_t is not None else None)
        u8, i64 = torch.uint8, torch.int64
        n = max(T_max * k, 1)
        self.ws = torch.empty(ep_workspace_bytes(T_max, E, k, H), dtype=u8, device=dev)
        self.send_x = torch.empty((n, H), dtype=u8, device=dev)
        self.send_sf = torch.empty((n, H // 32), dtype=u8, device=dev)
        self.send_eid = torch.empty(n, dtype=i64, device=dev)
        self.send_counts = torch.empty(self.ranks, dtype=i64, device=dev)
        m = max(self.recv_max, 1)
        self.recv_x = torch.empty((m, H), dtype=u8, device=dev)
        self.recv_sf = torch.empty((m, H // 32), dtype=u8, device=dev)
        self.recv_eid = torch.empty((m, 1), dtype=i64, device=dev)
        self.ones = torch.ones((m, 1), dtype=torch.float32, device=dev)
        self.y_loc = torch.empty((m, H), dtype=torch.bfloat16, device=dev)
        self.y_back = torch.empty((n, H), dtype=torch.bfloat16, device=dev)
        self.ws_loc = torch.empty(workspace_bytes(self.recv_max, self.E_loc, 1, H, I), dtype=u8, device=dev)
        # error words start clean (a step with no received rows runs no layer on ws_loc)
        self.ws[:4].zero_()
        self.ws_loc[:4].zero_()
        self.last_n_recv = 0  # rows the expert layer ran over in the last step

    # ---------------------------------------------------------------- phases
    def dispatch(self, x_fp8, x_sf, topk_idx, stream=None):
        """Step 1: fills send_x / send_sf / send_eid (rows grouped by destination
        rank) and returns send_counts (i64 [ranks], device)."""
        if x_fp8.shape[0] > self.T_max:
            raise ValueError(f"{x_fp8.shape[0]} tokens > T_max = {self.T_max}")
        ep_dispatch(x_fp8, x_sf, topk_idx, self.E, self.ranks, self.ws, self.send_x, self.send_sf, self.send_eid,
                    self.send_counts, stream=stream)
        return self.send_counts

    def expert(self, n: int, x=None, sf=None, eid=None, out=None, stream=None):
        """Step 3: the expert layer over n rows (default: the first n received
        rows; x u8 [>=n, H], sf u8 [>=n, H/32], eid i64 [>=n] local expert
        ids); returns their bf16 outputs ([n, H], a view of ``out``, default
        y_loc)."""
        n = int(n)
        if n > self.recv_max:
            raise ValueError(f"{n} rows > recv_max = {self.recv_max}")
        x = self.recv_x if x is None else x
        sf = self.recv_sf if sf is None else sf
        eid = self.recv_eid[:, 0] if eid is None else eid
        out = self.y_loc if out is None else out
        if n == 0:
            return out[:0]
        return forward(x[:n], sf[:n], eid[:n].view(n, 1), self.ones[:n], self.l1_t, self.l2_t, self.E_loc, self.H,
                       self.I, out=out[:n], workspace=self.ws_loc, stream=stream)

    def combine(self, topk_w, out=None, stream=None):
        """Step 5: out (bf16 [T, H]) from the returned rows in y_back."""
        return ep_combine(self.y_back, topk_w, self.E, self.ws, out=out, stream=stream)

    # ------------------------------------------------------------- peer memory
    def enable_peers(self, ipc=None):
        """Maps every rank's receive buffers and expert-layer output into this
        rank's address space (a collective over the group; see PeerBuffers)."""
        self.peers = PeerBuffers({"x": self.recv_x, "sf": self.recv_sf, "eid": self.recv_eid, "y": self.y_loc},
                                 group=self.group, ipc=ipc)
        self._flag = torch.zeros(1, dtype=torch.float32, device=self.recv_x.device)
        return self.peers

    def _barrier(self):
        # stream-ordered: work enqueued after it on this rank's stream starts
        # only once every rank has reached it
        import torch.distributed as dist
        dist.all_reduce(self._flag, group=self.group)

    def _route(self, topk_idx):
        return ep_route(topk_idx, self.E, self.H, self.ranks, self.ws, self.send_counts)

    def _push(self, x_fp8, x_sf, topk_idx, recv_base):
        t = self.peers.tables
        ep_dispatch_peers(x_fp8, x_sf, topk_idx, self.E, self.ws, t["x"], t["sf"], t["eid"], recv_base)

    def _pull(self, topk_idx, topk_w, recv_base, out):
        return ep_combine_peers(self.peers.tables["y"], recv_base, topk_idx, topk_w, self.E, self.H, self.ws,
                                out=out)

    def forward_peers(self, x_fp8, x_sf, topk_idx, topk_w, out=None):
        """One layer step over peer memory (after ``enable_peers`` on every
        rank); the same result as ``forward`` bit for bit."""
        import torch.distributed as dist
        if getattr(self, "peers", None) is None:
            raise RuntimeError("enable_peers() first (on every rank)")
        if x_fp8.shape[0] > self.T_max:
            raise ValueError(f"{x_fp8.shape[0]} tokens > T_max = {self.T_max}")
        counts = self._route(topk_idx)
        rows = [torch.empty_like(counts) for _ in range(self.ranks)]
        dist.all_gather(rows, counts, group=self.group)
        matrix = torch.stack(rows).tolist()
        most = max(sum(matrix[src][dst] for src in range(self.ranks)) for dst in range(self.ranks))
        if most > self.recv_max:
            raise ValueError(f"a rank would receive {most} rows > recv_max = {self.recv_max}")
        # this rank's first row in rank d's receive buffers: what ranks 0..rank-1 send to d
        base = [sum(matrix[src][d] for src in range(self.rank)) for d in range(self.ranks)]
        recv_base = torch.tensor(base, dtype=torch.int64, device=counts.device)
        n_recv = sum(matrix[src][self.rank] for src in range(self.ranks))
        self.last_n_recv = n_recv
        self._push(x_fp8, x_sf, topk_idx, recv_base)
        self._barrier()   # every rank's rows are in every receive buffer
        self.expert(n_recv)
        self._barrier()   # every rank's expert outputs are complete
        out = self._pull(topk_idx, topk_w, recv_base, out)
        self._barrier()   # nobody still reads a rank's buffers when the next step writes them
        return out

    def check(self, stream=None) -> int:
        """Synchronises the stream and returns the device status of the last
        step: the dispatch workspace's error word (dropped expert ids) or, if
        that is clean, the expert layer's (its bounded waits record timeouts
        there); 0 when both are clean."""
        st = check_device_error(self.ws, stream=stream)
        return st if st != 0 else check_device_error(self.ws_loc, stream=stream)

    # ------------------------------------------------------------- one step
    def _exchange(self, dst, src, out_splits, in_splits):
        import torch.distributed as dist
        dist.all_to_all_single(dst, src, output_split_sizes=out_splits, input_split_sizes=in_splits,
                               group=self.group)

    def forward(self, x_fp8, x_sf, topk_idx, topk_w, out=None):
        """One layer step on this rank's tokens; returns out (bf16 [T, H])."""
        for t, dt, name in ((x_fp8, torch.uint8, "x_fp8"), (x_sf, torch.uint8, "x_sf"),
                            (topk_idx, torch.int64, "topk_idx"), (topk_w, torch.float32, "topk_w")):
            if not isinstance(t, torch.Tensor) or t.dtype != dt or not t.is_contiguous():
                raise TypeError(f"{name} must be a contiguous {dt} tensor")
        counts = self.dispatch(x_fp8, x_sf, topk_idx)
        if self.ranks == 1:
            # no exchange: the expert layer reads the send buffers and writes
            # the rows combine reads
            self.last_n_recv = int(counts[0].item())
            self.expert(self.last_n_recv, self.send_x, self.send_sf, self.send_eid, out=self.y_back)
            return self.combine(topk_w, out=out)
        import torch.distributed as dist
        # every rank gets the whole [ranks, ranks] count matrix (row = source),
        # so that all ranks see an overflow of any rank's receive buffers and
        # stop together (recv_max must be the same on every rank)
        rows = [torch.empty_like(counts) for _ in range(self.ranks)]
        dist.all_gather(rows, counts, group=self.group)
        matrix = torch.stack(rows).tolist()
        send_splits = matrix[self.rank]
        recv_splits = [matrix[src][self.rank] for src in range(self.ranks)]
        n_send, n_recv = sum(send_splits), sum(recv_splits)
        most = max(sum(matrix[src][dst] for src in range(self.ranks)) for dst in range(self.ranks))
        if most > self.recv_max:
            raise ValueError(f"a rank would receive {most} rows > recv_max = {self.recv_max}")
        self.last_n_recv = n_recv
        self._exchange(self.recv_x[:n_recv], self.send_x[:n_send], recv_splits, send_splits)
        self._exchange(self.recv_sf[:n_recv], self.send_sf[:n_send], recv_splits, send_splits)
        self._exchange(self.recv_eid[:n_recv, 0], self.send_eid[:n_send], recv_splits, send_splits)
        y = self.expert(n_recv)
        # bf16 rows travel as bytes (2H per row), which every backend moves
        self._exchange(self.y_back[:n_send].view(torch.uint8), y.view(torch.uint8), send_splits, recv_splits)
        return self.combine(topk_w, out=out)

    __call__ = forward
