"""GPU parity of the whole layer (moe_forward through the C ABI) against the
oracle, element by element per token row: rel L2 <= 1e-2 and max abs <=
5e-2 * max|row| (the tolerance the layer is specified with).  Small cases are
checked on every token; the full-size workloads on sampled tokens, each of
which the oracle evaluates exactly (a token's output depends only on its own
row and its experts)."""
import gc

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from cases import compare_rows, experts_of, gpu_layer, oracle_side

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def run_and_compare(moe, w, routing=None, tokens=None, gen_device="cuda", check_repeat=True, situ=None):
    """situ: None (SwiGLU) or (beta, linear_beta or None)."""
    g = gpu_layer(w, routing=routing, gen_device=gen_device)
    ws = torch.empty(moe.workspace_bytes(w.T, w.E, w.k, w.H, w.I), dtype=torch.uint8, device="cuda")
    act = None if situ is None else moe.activation("situ", situ[0], situ[1])
    out = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I, workspace=ws,
                      act=act)
    status = moe.check_device_error(ws)
    idx = g["idx"].cpu().numpy()
    if check_repeat:
        out2 = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I, workspace=ws,
                           act=act)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "not deterministic"
    tok = np.arange(w.T) if tokens is None else np.asarray(tokens)
    xq, xs, ex = oracle_side(w, g["x"], g["idx"], experts_of(idx, tok, w.E), gen_device=gen_device)
    kw = {} if situ is None else dict(activation="situ", beta=situ[0], linear_beta=situ[1])
    ref = oracle.forward(xq, xs, idx, g["tw"].cpu().numpy(), ex, w.E, w.H, w.I,
                         tokens=None if tokens is None else tok.astype(np.int32), **kw)
    worst = compare_rows(out[torch.as_tensor(tok, device="cuda")], ref["out_bf16"], w.name)
    del g, ws, out
    gc.collect()
    torch.cuda.empty_cache()
    return status, worst


SMALL = [
    W.WORKLOADS[0],
    W.custom("ragged", T=37, E=5, k=3, H=384, I=256, seed=21),              # chunk rows not /16
    W.custom("multichunk", T=300, E=2, k=2, H=256, I=128, seed=22),         # experts with > 128 rows
    W.custom("k_eq_E", T=20, E=4, k=4, H=256, I=384, seed=23),
    W.custom("one_token", T=1, E=16, k=4, H=512, I=256, seed=24),
    W.custom("wide", T=33, E=3, k=2, H=1024, I=1024, seed=25),
    W.custom("zipf_small", T=512, E=32, k=4, H=256, I=256, seed=26, routing="zipf"),
    W.custom("max_E_one_block", T=300, E=1024, k=2, H=128, I=128, seed=43),   # 1024 experts, one-block routing
    W.custom("max_E_multi_block", T=2000, E=1024, k=2, H=128, I=128, seed=45),  # 1024 experts, block-scan routing
    W.custom("max_I", T=20, E=2, k=2, H=256, I=8192, seed=44),                # largest intermediate size
    W.custom("k10", T=40, E=12, k=10, H=256, I=128, seed=46),                 # top-k above the combine's batch of 8
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_layer_small_all_tokens(moe, w):
    status, _ = run_and_compare(moe, w)
    assert status == 0


def test_layer_single_expert_all_tokens_many_chunks(moe):
    w = W.custom("hot", T=700, E=3, k=1, H=256, I=256, seed=27)
    idx = torch.full((w.T, 1), 1, dtype=torch.int64)
    tw = torch.ones((w.T, 1), dtype=torch.float32)
    status, _ = run_and_compare(moe, w, routing=(idx, tw))
    assert status == 0


def test_layer_structured_routing(moe):
    w = W.custom("structured", T=96, E=12, k=4, H=256, I=256, seed=28)
    status, _ = run_and_compare(moe, w, routing=W.structured_routing(w.T, w.k, w.E))
    assert status == 0


def test_layer_duplicate_and_dropped_slots(moe):
    w = W.custom("dup_drop", T=24, E=6, k=3, H=256, I=256, seed=29)
    idx, tw = W.gen_routing(w)
    idx[0, 1] = idx[0, 0]        # same expert twice
    idx[5, 2] = 99               # dropped
    idx[7] = -1                  # a token with every slot dropped
    status, _ = run_and_compare(moe, w, routing=(idx, tw))
    assert status == 5  # MOE_ERR_BAD_ROUTING is reported, the rest is computed


def split_of(idx, w, gemm1, mx=True):
    """Units per leftover item the 32-row GEMMs cut their incomplete last round
    into (0: none), for asserting that a case exercises that path: grid =
    min(item bound, SMs), leftover = items % grid, split = min(min(grid, 256) //
    leftover, stages per item) when at least 2."""
    R = idx.size
    counts = np.bincount(idx[idx >= 0].ravel(), minlength=w.E)
    chunks = int(sum((c + 31) // 32 for c in counts))
    per_chunk = w.I // 128 if gemm1 else (w.H // 128 + 1) // 2
    max_chunks = (R + 31) // 32 + min(R, w.E)
    grid = min(max_chunks * per_chunk, torch.cuda.get_device_properties(0).multi_processor_count)
    K = w.H if gemm1 else w.I
    n_steps = K // 256 if not mx else (K // 128 + 1) // 2
    rem = chunks * per_chunk % grid
    if rem == 0:
        return 0
    S = min(min(grid, 256) // rem, n_steps)
    return S if S >= 2 else 0


def one_expert_routing(w, experts):
    """Slot j of every token goes to experts[j]; positive normalised weights."""
    idx = torch.tensor([experts] * w.T, dtype=torch.int64)
    tw = torch.rand((w.T, w.k), generator=torch.Generator().manual_seed(w.seed)) + 0.1
    return idx, (tw / tw.sum(1, keepdim=True)).float()


SPLIT = [
    # one chunk: every item is cut along K (4 units of one stage each)
    (W.custom("split_even", T=32, E=64, k=1, H=1024, I=1024, seed=47), [5]),
    # two chunks; an odd number of K blocks leaves a last unit with one block,
    # and GEMM2's last item holds one tile
    (W.custom("split_odd_kb", T=20, E=64, k=2, H=640, I=384, seed=48), [3, 9]),
    # whole rounds first, then the leftover items cut into units
    (W.custom("split_mixed", T=32, E=64, k=2, H=1024, I=1024, seed=49), None),
]


@pytest.mark.parametrize("w,experts", SPLIT, ids=lambda c: getattr(c, "name", ""))
def test_layer_split_units(moe, w, experts):
    """Items of an incomplete last round split along K across CTAs, their
    partial accumulators added by the last unit: same results as the oracle,
    and deterministic."""
    routing = one_expert_routing(w, experts) if experts else W.gen_routing(w)
    ic = routing[0].numpy()
    assert split_of(ic, w, True) >= 2 and split_of(ic, w, False) >= 2, "case does not split"
    status, _ = run_and_compare(moe, w, routing=routing)
    assert status == 0


def side_list_routing(w, counts, seed):
    """Routing with the given rows per expert (T*k in total), slots shuffled."""
    ids = np.repeat(np.arange(len(counts)), counts)
    assert ids.size == w.T * w.k
    np.random.default_rng(seed).shuffle(ids)
    idx = torch.as_tensor(ids.reshape(w.T, w.k), dtype=torch.int64)
    tw = torch.rand((w.T, w.k), generator=torch.Generator().manual_seed(seed)) + 0.1
    return idx, (tw / tw.sum(1, keepdim=True)).float()


# T*k > 8E: 160-row chunks for the main list; experts with at most 32 rows
# (here 32, 31 and 1; two experts get none) go to the side list of 32-row chunks
SIDE_COUNTS = [32, 33, 1, 0, 31, 60, 43, 0]


def test_layer_side_list(moe):
    """Both chunk lists in one forward: the boundary loads (32 rows: side; 33:
    main), an expert with one row and experts with none."""
    w = W.custom("side_list", T=100, E=8, k=2, H=384, I=256, seed=61)
    status, _ = run_and_compare(moe, w, routing=side_list_routing(w, SIDE_COUNTS, 61))
    assert status == 0


def test_layer_decode_full(moe):
    w = W.WORKLOADS[1]            # T=8, E=384, k=6, H=7168, I=3072: every token
    status, _ = run_and_compare(moe, w)
    assert status == 0


@pytest.mark.parametrize("cfg,ntok", [(2, 12), (3, 8), (4, 8)])
def test_layer_full_size_sampled(moe, cfg, ntok):
    w = W.WORKLOADS[cfg]
    idx, tw = W.gen_routing(w, "cuda")
    ic = idx.cpu().numpy()
    rng = np.random.default_rng(cfg)
    tokens = set(rng.choice(w.T, ntok - 2, replace=False).tolist()) | {0, w.T - 1}
    if cfg == 4:
        # include tokens of the hottest expert, whose rows span many chunks
        hot = np.bincount(ic.ravel(), minlength=w.E).argmax()
        users = np.nonzero((ic == hot).any(axis=1))[0]
        tokens |= {int(users[0]), int(users[len(users) // 2]), int(users[-1])}
    status, _ = run_and_compare(moe, w, routing=(idx, tw), tokens=sorted(tokens), check_repeat=False)
    assert status == 0


def test_expert_stats_accumulate(moe):
    w = W.custom("stats", T=40, E=8, k=2, H=128, I=128, seed=30)
    g = gpu_layer(w)
    stats = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    for _ in range(3):
        moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I, expert_stats=stats)
    ref = np.bincount(g["idx"].cpu().numpy().ravel(), minlength=w.E) * 3
    assert np.array_equal(stats.cpu().numpy(), ref)


def test_stage_events_and_stream(moe):
    w = W.WORKLOADS[0]
    g = gpu_layer(w)
    s = torch.cuda.Stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(moe.NUM_STAGE_EVENTS)]
    with torch.cuda.stream(s):
        out = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I,
                          events=ev, stream=s)
    s.synchronize()
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(moe.NUM_STAGE_EVENTS - 1)]
    assert all(t >= 0 for t in times)
    ref = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


SITU_CASES = [(W.WORKLOADS[0], (1.25, 1.5)), (W.custom("situ_ragged", T=37, E=5, k=3, H=384, I=256, seed=41), (0.5, None)),
              (W.custom("situ_multichunk", T=300, E=2, k=2, H=256, I=128, seed=42), (3.0, 0.75))]


@pytest.mark.parametrize("w,coef", SITU_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_layer_situ_small(moe, w, coef):
    status, _ = run_and_compare(moe, w, situ=coef)
    assert status == 0


def test_layer_situ_decode_full(moe):
    status, _ = run_and_compare(moe, W.WORKLOADS[1], situ=(1.25, 1.5))
    assert status == 0


def test_layer_situ_prefill_sampled(moe):
    w = W.WORKLOADS[3]
    idx, tw = W.gen_routing(w, "cuda")
    tokens = sorted(set(np.random.default_rng(5).choice(w.T, 6, replace=False).tolist()) | {0, w.T - 1})
    status, _ = run_and_compare(moe, w, routing=(idx, tw), tokens=tokens, check_repeat=False, situ=(1.25, None))
    assert status == 0
