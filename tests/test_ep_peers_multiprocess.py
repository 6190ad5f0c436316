"""The peer-memory step of the expert-parallel layer (ExpertParallelLayer.
enable_peers / forward_peers) on CPU with gloo at world sizes 2 and 4.

What runs for real: the buffer export, the all-gather of (handle, offset)
records, the opening of every other rank's allocation once, the address
tables, the count exchange, this rank's first row in every receive buffer
(recv_base), the barriers and the expert phase's row counts.  What is stood
in for: CUDA IPC by shared files (one file per rank holds its receive and
output buffers, so buffers sit at non-zero offsets of one allocation, as
with a framework allocator), and the push / pull kernels by their
definitions in numpy, writing and reading through the exchanged addresses;
the expert phase is the oracle over this rank's experts only.  Every rank's
output must equal, bit for bit, the combine of the bf16-rounded expert
outputs the oracle computes with all experts at hand."""
import os
import sys
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "tests"))
import test_ep_multiprocess as M  # noqa: E402

E, K, H, I = M.E, M.K, M.H, M.I


class FileIpc:
    """Stand-in for CUDA IPC: an 'allocation' is a shared file; a handle is
    its path; opening maps the file and returns a fake base address."""

    def __init__(self):
        self.maps = {}      # base -> (numpy uint8 array over the file)
        self.opened, self.closed = [], []
        self.next_base = 1 << 44

    def register_local(self, arr):
        self.maps[arr.ctypes.data] = arr

    def export(self, t):
        for base, arr in self.maps.items():
            if base <= t.data_ptr() < base + arr.size:
                path = arr.filename.encode()
                return path.ljust(64, b"\0"), t.data_ptr() - base
        raise AssertionError("buffer outside the shared file")

    def open(self, handle, device):
        path = handle.rstrip(b"\0").decode()
        arr = np.memmap(path, dtype=np.uint8, mode="r+")
        base = self.next_base
        self.next_base += 1 << 36
        self.maps[base] = arr
        self.opened.append((path, device))
        return base

    def close(self, base):
        self.closed.append(base)

    def view(self, addr, nbytes):
        for base, arr in self.maps.items():
            if base <= addr and addr + nbytes <= base + arr.size:
                return arr[addr - base:addr - base + nbytes]
        raise AssertionError(f"address {addr:#x} maps nowhere")


def _peer_layer_class():
    import ep_definition as D
    base_cls = M._fake_layer_class()

    class PeerPhases(base_cls):
        def _route(self, topk_idx):
            self.plan = D.dispatch_plan(topk_idx.numpy(), self.E, self.ranks)
            self.send_counts.copy_(torch.from_numpy(self.plan[1]))
            return self.send_counts

        def _dest(self):
            order, counts, eid, inv = self.plan
            dest = np.repeat(np.arange(self.ranks), counts)      # rows are grouped by destination rank
            pos = np.arange(order.size) - np.concatenate([[0], np.cumsum(counts)[:-1]])[dest]
            return order, eid, inv, dest, pos

        def _push(self, x_fp8, x_sf, topk_idx, recv_base):
            order, eid, _, dest, pos = self._dest()
            t = {n: v.tolist() for n, v in self.peers.tables.items()}
            for i, slot in enumerate(order):
                d, row = int(dest[i]), int(recv_base[dest[i]]) + int(pos[i])
                tok = int(slot) // self.k
                self.ipc.view(t["x"][d] + row * H, H)[:] = x_fp8[tok].numpy()
                self.ipc.view(t["sf"][d] + row * (H // 32), H // 32)[:] = x_sf[tok].numpy()
                self.ipc.view(t["eid"][d] + row * 8, 8)[:] = np.frombuffer(np.int64(eid[i]).tobytes(), np.uint8)

        def _pull(self, topk_idx, topk_w, recv_base, out):
            order, _, inv, dest, pos = self._dest()
            t = self.peers.tables["y"].tolist()
            rows = np.zeros((order.size, H), np.float32)
            for i in range(order.size):
                d, row = int(dest[i]), int(recv_base[dest[i]]) + int(pos[i])
                raw = self.ipc.view(t[d] + row * 2 * H, 2 * H).view(np.uint16).astype(np.uint32) << 16
                rows[i] = raw.view(np.float32)
            return D.combine(rows, inv, topk_w.numpy(), self.k)

        def _barrier(self):
            import torch.distributed as dist
            dist.barrier(group=self.group)

    return PeerPhases


def _worker(rank, world, port, q, tokens, tmp):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T = tokens[rank]
        xq, xs, idx, tw, experts = M._inputs(rank, T)
        layer = _peer_layer_class()(None, None, E, K, H, I, T_max=max(tokens), device="cpu")
        e_loc = E // world
        layer.experts = {e: m for e, m in experts.items() if e // e_loc == rank}
        # this rank's receive and output buffers: views of one shared file, 256-byte aligned pieces
        m = layer.recv_max
        sizes = {"x": m * H, "sf": m * (H // 32), "eid": m * 8, "y": m * H * 2}
        offs, o = {}, 256              # nothing at offset 0: the offsets must travel
        for n in ("x", "sf", "eid", "y"):
            offs[n] = o
            o += (sizes[n] + 255) // 256 * 256
        arr = np.memmap(os.path.join(tmp, f"rank{rank}.buf"), dtype=np.uint8, mode="w+", shape=(o,))
        view = lambda n, dt, shape: torch.from_numpy(arr[offs[n]:offs[n] + sizes[n]]).view(dt).view(shape)
        layer.recv_x = view("x", torch.uint8, (m, H))
        layer.recv_sf = view("sf", torch.uint8, (m, H // 32))
        layer.recv_eid = view("eid", torch.int64, (m, 1))
        layer.y_loc = view("y", torch.bfloat16, (m, H))
        layer.ipc = FileIpc()
        layer.ipc.register_local(arr)
        peers = layer.enable_peers(ipc=layer.ipc)
        tables = {n: v.tolist() for n, v in peers.tables.items()}
        # own entries are this rank's own addresses; every other rank's file is opened once
        own_ok = all(tables[n][rank] == getattr(layer, b).data_ptr()
                     for n, b in (("x", "recv_x"), ("sf", "recv_sf"), ("eid", "recv_eid"), ("y", "y_loc")))
        opened = sorted(os.path.basename(p) for p, _ in layer.ipc.opened)
        want_opened = sorted(f"rank{d}.buf" for d in range(world) if d != rank)
        offsets_ok = all(tables[n][d] - tables["x"][d] == offs[n] - offs["x"]
                         for n in ("sf", "eid", "y") for d in range(world))
        outs = []
        for _ in range(2):  # two steps in a row: buffers reused
            outs.append(layer.forward_peers(torch.from_numpy(xq), torch.from_numpy(xs), idx, tw))
        want = M._expected(xq, xs, idx, tw, experts, world)
        same = all(o.shape == want.shape and torch.equal(o.view(torch.int16), want.view(torch.int16)) for o in outs)
        peers.close()
        q.put((rank, dict(same=bool(same), own=own_ok, opened=opened == want_opened, offsets=offsets_ok,
                          closed=len(layer.ipc.closed) == world - 1)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("tokens", [(12, 7), (9, 0, 5, 3)], ids=["two_ranks", "four_ranks_one_idle"])
def test_peer_step_matches_single_rank_definition(tokens):
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = M.free_port()
    with tempfile.TemporaryDirectory() as tmp:
        procs = [ctx.Process(target=_worker, args=(r, world, port, q, tokens, tmp)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res = dict(q.get(timeout=5) for _ in range(world))
    good = dict(same=True, own=True, opened=True, offsets=True, closed=True)
    assert res == {r: good for r in range(world)}, res
