"""The exchange of the expert-parallel layer (ExpertParallelLayer.forward) on
CPU with gloo at world sizes 2 and 4: the count all-gather, the row all-to-alls in
both directions and their split sizes, every rank taking the same collective
steps whatever its token count, and an overflow of the receive buffers
stopping both ranks.  The three CUDA phases (dispatch, expert layer, combine)
are replaced by their definitions on CPU (numpy and the oracle); the expert
phase is given only its own rank's experts, so a row delivered to the wrong
rank fails the oracle's lookup.  Each rank's output must equal, bit for bit,
the combine of the bf16-rounded expert outputs that the oracle computes for
that rank's tokens with all experts at hand."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, K, H, I = 8, 2, 128, 128


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_layer_class():
    import ep_definition as D
    import oracle
    from moe_expert_layer_08_b200.ep import ExpertParallelLayer

    class CpuPhases(ExpertParallelLayer):
        experts = None

        def dispatch(self, x_fp8, x_sf, topk_idx, stream=None):
            order, counts, eid, inv = D.dispatch_plan(topk_idx.numpy(), self.E, self.ranks)
            n, t = order.size, torch.from_numpy(order // self.k)
            self.send_x[:n] = x_fp8[t]
            self.send_sf[:n] = x_sf[t]
            self.send_eid[:n] = torch.from_numpy(eid)
            self.send_counts.copy_(torch.from_numpy(counts))
            self.inv = inv
            return self.send_counts

        def expert(self, n, x=None, sf=None, eid=None, out=None, stream=None):
            x = self.recv_x if x is None else x
            sf = self.recv_sf if sf is None else sf
            eid = self.recv_eid[:, 0] if eid is None else eid
            out = self.y_loc if out is None else out
            if n == 0:
                return out[:0]
            ids = eid[:n].numpy() + self.rank * self.E_loc
            res = oracle.forward(x[:n].numpy(), sf[:n].numpy(), ids[:, None], np.ones((n, 1), np.float32),
                                 self.experts, self.E, self.H, self.I)
            out[:n].view(torch.int16).copy_(torch.from_numpy(res["out_bf16"].view(np.int16)))
            return out[:n]

        def combine(self, topk_w, out=None, stream=None):
            n = int(self.send_counts.sum())
            return D.combine(self.y_back[:n].float().numpy(), self.inv, topk_w.numpy(), self.k)

    return CpuPhases


def _inputs(rank, T):
    import oracle
    import workloads as W
    wt = W.custom("ep_weights", T=1, E=E, k=K, H=H, I=I, seed=60)      # the same experts on every rank
    wx = W.custom(f"ep_tokens{rank}", T=max(T, 1), E=E, k=K, H=H, I=I, seed=61 + rank)
    x = W.gen_x(wx, "cpu")[:T]
    idx, tw = (a[:T].contiguous() for a in W.gen_routing(wx, "cpu"))
    if T >= 2:
        idx[0, 1] = E            # a dropped slot
        idx[1, :] = 5            # the same expert twice
    xq, xs = oracle.quantize_e4m3(x.float().numpy())
    experts = {}
    for e in range(E):
        a, b = oracle.quantize_e2m1(W.gen_l1(wt, e, "cpu").float().numpy())
        c, d = oracle.quantize_e2m1(W.gen_l2(wt, e, "cpu").float().numpy())
        experts[e] = (a, b, c, d)
    return xq, xs, idx, tw, experts


def _expected(xq, xs, idx, tw, experts, ranks):
    """The combine of the bf16-rounded expert outputs the oracle computes for
    these tokens with every expert at hand."""
    import ep_definition as D
    import oracle
    if idx.shape[0] == 0:
        return torch.empty((0, H), dtype=torch.bfloat16)
    y = oracle.forward(xq, xs, idx.numpy(), tw.numpy(), experts, E, H, I, intermediates=True)["y"]
    order, _, _, inv = D.dispatch_plan(idx.numpy(), E, ranks)
    rows = torch.from_numpy(y[order // K, order % K]).to(torch.bfloat16).float().numpy()
    return D.combine(rows, inv, tw.numpy(), K)


def _worker(rank, world, port, q, tokens, recv_max):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T = tokens[rank]
        xq, xs, idx, tw, experts = _inputs(rank, T)
        layer = _fake_layer_class()(None, None, E, K, H, I, T_max=max(tokens), recv_max=recv_max, device="cpu")
        e_loc = E // world
        layer.experts = {e: m for e, m in experts.items() if e // e_loc == rank}
        try:
            out = layer.forward(torch.from_numpy(xq), torch.from_numpy(xs), idx, tw)
        except ValueError as err:
            q.put((rank, "ValueError", str(err)))
            return
        want = _expected(xq, xs, idx, tw, experts, world)
        same = out.shape == want.shape and torch.equal(out.view(torch.int16), want.view(torch.int16))
        q.put((rank, "ok", bool(same)))
    finally:
        dist.destroy_process_group()


def _run(tokens, recv_max=None):
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, tokens, recv_max)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    return {r: (kind, val) for r, kind, val in (q.get(timeout=5) for _ in range(world))}


@pytest.mark.parametrize("tokens", [(12, 7), (9, 0), (5, 0, 12, 3)], ids=["uneven", "one_rank_idle", "four_ranks"])
def test_exchange_matches_single_rank_definition(tokens):
    res = _run(tokens)
    assert res == {r: ("ok", True) for r in range(len(tokens))}, res


def test_receive_overflow_stops_every_rank():
    res = _run((12, 7), recv_max=3)
    assert {r: kind for r, (kind, _) in res.items()} == {0: "ValueError", 1: "ValueError"}, res


def test_one_rank_runs_without_exchange():
    """Without a process group the layer is one rank: no collective, the
    expert phase reads the send buffers and writes the rows combine reads."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    xq, xs, idx, tw, experts = _inputs(0, 11)
    layer = _fake_layer_class()(None, None, E, K, H, I, T_max=11, device="cpu")
    assert layer.ranks == 1 and layer.E_loc == E
    layer.experts = experts
    out = layer.forward(torch.from_numpy(xq), torch.from_numpy(xs), idx, tw)
    want = _expected(xq, xs, idx, tw, experts, 1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    assert layer.last_n_recv == int((idx.numpy() < E).sum())
