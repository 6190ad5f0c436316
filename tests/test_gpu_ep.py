"""Expert parallelism through the C ABI on one GPU (moe_ep_dispatch, the
layer with k = 1 over each rank's experts, moe_ep_combine).

* One rank (ExpertParallelLayer.forward, no exchange): the output equals
  moe_forward's bit for bit (the same rows reach the same GEMM work in the
  same order, and the layer's k = 1, weight-1 combine passes the bf16 rows
  through unchanged).
* Two and four ranks emulated in one process: every rank's dispatch, then
  the exchange done by the test as copies between the ranks' buffers (no
  collective, no kernel that waits on another rank), every rank's expert
  layer, the copies back, every rank's combine; and the combine over peer
  memory (moe_ep_combine_peers), reading each row from the buffer of the
  rank that computed it, equal to the combine of the returned rows bit for
  bit; and the dispatch over peer memory (moe_ep_route, then
  moe_ep_dispatch_peers writing into every rank's receive buffers), equal to
  what the exchange of the send buffers delivered.  The dispatch outputs (row
  counts per rank, local expert ids, rows and scales in routing order) are
  compared bit for bit with the definition; each rank's output with the
  oracle within the layer's tolerance and with moe_forward over all experts.
"""
import numpy as np
import pytest
import torch

import ep_definition as D
import oracle
import workloads as W
from cases import compare_rows, experts_of, gpu_layer, oracle_side

pytestmark = pytest.mark.gpu
DEVICE = "cuda"


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def shard(t, r, n_ranks):
    per = t.numel() // n_ranks
    return t[r * per:(r + 1) * per]


@pytest.mark.parametrize("w", [W.custom("ep1_small_chunks", T=20, E=8, k=2, H=256, I=256, seed=70),
                               W.custom("ep1_large_chunks", T=300, E=8, k=3, H=256, I=128, seed=71)],
                         ids=lambda w: w.name)
def test_one_rank_equals_moe_forward_bitwise(moe, w):
    from moe_expert_layer_08_b200.ep import ExpertParallelLayer
    g = gpu_layer(w)
    ref = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I)
    layer = ExpertParallelLayer(g["l1_t"], g["l2_t"], w.E, w.k, w.H, w.I, T_max=w.T)
    assert layer.ranks == 1
    out = layer(g["xq"], g["xs"], g["idx"], g["tw"])
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert moe.check_device_error(layer.ws) == 0


def run_emulated(moe, n_ranks, tokens, w_weights, drop=True):
    """Returns per rank (inputs, output) after the five phases on one GPU."""
    from moe_expert_layer_08_b200.ep import ExpertParallelLayer
    E, k, H, I = w_weights.E, w_weights.k, w_weights.H, w_weights.I
    g = gpu_layer(W.custom("ep_w", T=1, E=E, k=k, H=H, I=I, seed=w_weights.seed))
    ranks = []
    for r, T in enumerate(tokens):
        wx = W.custom(f"ep_tok{r}", T=max(T, 1), E=E, k=k, H=H, I=I, seed=w_weights.seed + 1 + r)
        x = W.gen_x(wx, DEVICE)[:T].contiguous()
        idx, tw = (a[:T].contiguous() for a in W.gen_routing(wx, DEVICE))
        if drop and T >= 2:
            idx[0, k - 1] = E + 3       # a dropped slot
            idx[1, :] = E - 1           # one expert, every slot
        xq, xs = moe.quantize_fp8(x) if T > 0 else (torch.empty((0, H), dtype=torch.uint8, device=DEVICE),
                                                    torch.empty((0, H // 32), dtype=torch.uint8, device=DEVICE))
        layer = ExpertParallelLayer(shard(g["l1_t"], r, n_ranks), shard(g["l2_t"], r, n_ranks), E, k, H, I,
                                    T_max=max(tokens), rank=r, ranks=n_ranks)
        ranks.append(dict(x=x, xq=xq, xs=xs, idx=idx, tw=tw, layer=layer))
    # 1. dispatch on every rank
    C = np.stack([rk["layer"].dispatch(rk["xq"], rk["xs"], rk["idx"]).cpu().numpy() for rk in ranks])
    for rk, c in zip(ranks, C):
        order, cnt, eid, inv = D.dispatch_plan(rk["idx"].cpu().numpy(), E, n_ranks)
        n = order.size
        L = rk["layer"]
        assert np.array_equal(c, cnt)
        assert np.array_equal(L.send_eid[:n].cpu().numpy(), eid)
        t = torch.as_tensor(order // k, device=DEVICE)
        assert torch.equal(L.send_x[:n], rk["xq"][t]) and torch.equal(L.send_sf[:n], rk["xs"][t])
        if rk["x"].shape[0] > 0:  # T = 0 enqueues no routing: the word is not written
            assert moe.check_device_error(L.ws) == (5 if drop and rk["x"].shape[0] >= 2 else 0)
    # 2. rows to their ranks (source-major), 3. the expert layer on every rank
    off = np.concatenate([np.zeros((n_ranks, 1), np.int64), np.cumsum(C, axis=1)], axis=1)   # [src, dst+1]
    ys = []
    for d, rk in enumerate(ranks):
        L, at = rk["layer"], 0
        for s, src in enumerate(ranks):
            a, b = int(off[s, d]), int(off[s, d] + C[s, d])
            L.recv_x[at:at + b - a] = src["layer"].send_x[a:b]
            L.recv_sf[at:at + b - a] = src["layer"].send_sf[a:b]
            L.recv_eid[at:at + b - a, 0] = src["layer"].send_eid[a:b]
            at += b - a
        ys.append(L.expert(at))
    # 4. rows back to their sources, 5. combine on every rank
    outs = []
    for s, rk in enumerate(ranks):
        for d in range(n_ranks):
            start = int(C[:s, d].sum())
            a, b = int(off[s, d]), int(off[s, d] + C[s, d])
            rk["layer"].y_back[a:b] = ys[d][start:start + b - a]
        outs.append(rk["layer"].combine(rk["tw"]))
    torch.cuda.synchronize()
    return g, ranks, outs, C


def check_peer_paths(moe, ranks, outs, C, ww):
    """The combine over peer memory (each rank reads its rows where the ranks'
    expert layers left them, here other buffers of the same GPU) equals the
    combine of the returned rows; the dispatch over peer memory (routing and
    counts, then every rank writing its rows into fresh receive buffers)
    delivers what the exchange of the send buffers delivered."""
    n_ranks = len(ranks)
    peer_y = torch.tensor([rk["layer"].y_loc.data_ptr() for rk in ranks], dtype=torch.int64, device=DEVICE)
    for r, (rk, out) in enumerate(zip(ranks, outs)):
        base = torch.tensor([int(C[:r, d].sum()) for d in range(n_ranks)], dtype=torch.int64, device=DEVICE)
        fused = moe.ep_combine_peers(peer_y, base, rk["idx"], rk["tw"], ww.E, ww.H, rk["layer"].ws)
        assert torch.equal(fused.view(torch.int16), out.view(torch.int16)), f"rank {r}"
    n_recv = C.sum(axis=0)
    u8 = dict(dtype=torch.uint8, device=DEVICE)
    bufs = [dict(x=torch.zeros((max(int(n), 1), ww.H), **u8), sf=torch.zeros((max(int(n), 1), ww.H // 32), **u8),
                 eid=torch.full((max(int(n), 1),), -1, dtype=torch.int64, device=DEVICE)) for n in n_recv]
    table = {key: torch.tensor([b[key].data_ptr() for b in bufs], dtype=torch.int64, device=DEVICE)
             for key in ("x", "sf", "eid")}
    for r, rk in enumerate(ranks):
        ws = torch.empty(moe.ep_workspace_bytes(rk["layer"].T_max, ww.E, ww.k, ww.H), **u8)
        counts = moe.ep_route(rk["idx"], ww.E, ww.H, n_ranks, ws)
        assert np.array_equal(counts.cpu().numpy(), C[r])
        base = torch.tensor([int(C[:r, d].sum()) for d in range(n_ranks)], dtype=torch.int64, device=DEVICE)
        moe.ep_dispatch_peers(rk["xq"], rk["xs"], rk["idx"], ww.E, ws, table["x"], table["sf"], table["eid"], base)
    torch.cuda.synchronize()
    for d, rk in enumerate(ranks):
        n, L = int(n_recv[d]), rk["layer"]
        assert torch.equal(bufs[d]["x"][:n], L.recv_x[:n]), f"rank {d} rows"
        assert torch.equal(bufs[d]["sf"][:n], L.recv_sf[:n]), f"rank {d} scales"
        assert torch.equal(bufs[d]["eid"][:n], L.recv_eid[:n, 0]), f"rank {d} expert ids"


@pytest.mark.parametrize("n_ranks,tokens", [(2, (37, 20)), (4, (64, 0, 9, 33))], ids=["R2", "R4_idle_rank"])
def test_emulated_ranks_match_oracle(moe, n_ranks, tokens):
    ww = W.custom("ep_weights", T=1, E=8, k=2, H=256, I=256, seed=80)
    g, ranks, outs, C = run_emulated(moe, n_ranks, tokens, ww)
    check_peer_paths(moe, ranks, outs, C, ww)
    for r, (rk, out) in enumerate(zip(ranks, outs)):
        T = rk["x"].shape[0]
        assert out.shape == (T, ww.H)
        if T == 0:
            continue
        idx = rk["idx"].cpu().numpy()
        xq, xs, ex = oracle_side(ww, rk["x"], rk["idx"], experts_of(idx, np.arange(T), ww.E), gen_device=DEVICE)
        ref = oracle.forward(xq, xs, idx, rk["tw"].cpu().numpy(), ex, ww.E, ww.H, ww.I)
        compare_rows(out, ref["out_bf16"], f"rank {r}")
        full = moe.forward(rk["xq"], rk["xs"], rk["idx"], rk["tw"], g["l1_t"], g["l2_t"], ww.E, ww.H, ww.I)
        compare_rows(out, oracle.f32_to_bf16(full.float().cpu().numpy()), f"rank {r} vs one GPU")


def test_emulated_ranks_decode_sizes(moe):
    """Eight ranks at the decode workload's sizes: 384 experts (48 per rank),
    8 tokens per rank, top-6, H = 7168, I = 3072.  Every rank against
    moe_forward over all experts, rank 0 against the oracle, and the
    peer-memory paths."""
    ww = W.custom("ep_decode", T=1, E=384, k=6, H=7168, I=3072, seed=90)
    g, ranks, outs, C = run_emulated(moe, 8, (8,) * 8, ww, drop=False)
    check_peer_paths(moe, ranks, outs, C, ww)
    for r, (rk, out) in enumerate(zip(ranks, outs)):
        full = moe.forward(rk["xq"], rk["xs"], rk["idx"], rk["tw"], g["l1_t"], g["l2_t"], ww.E, ww.H, ww.I)
        compare_rows(out, oracle.f32_to_bf16(full.float().cpu().numpy()), f"rank {r} vs one GPU")
    rk = ranks[0]
    idx = rk["idx"].cpu().numpy()
    xq, xs, ex = oracle_side(ww, rk["x"], rk["idx"], experts_of(idx, np.arange(8), ww.E), gen_device=DEVICE)
    ref = oracle.forward(xq, xs, idx, rk["tw"].cpu().numpy(), ex, ww.E, ww.H, ww.I)
    compare_rows(outs[0], ref["out_bf16"], "rank 0")
