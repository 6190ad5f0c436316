"""GPU parity of the BF16 shared expert (moe_shared_forward through the C ABI)
against the oracle, per token row: rel L2 <= 1e-2 and max abs <= 5e-2 *
max|row| (the DeepGEMM PR #416 test body bounds the shared output's relative
L2 by 1e-2).  Small cases on every token, with every token-block size (32-token
blocks up to T = 64, 64-token blocks up to 128, else 128-token blocks), with
and without a K split,
ragged token counts and an odd output-tile count;
the full-size case on sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from cases import compare_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def run_and_compare(moe, T, SH, SI, seed, tokens=None, situ=None, repeat=True):
    x, l1, l2 = W.gen_shared(T, SH, SI, seed, "cuda")
    act = None if situ is None else moe.activation("situ", situ[0], situ[1])
    ws = moe.shared_workspace(T, SH, SI, "cuda")
    y = moe.shared_forward(x, l1, l2, workspace=ws, act=act)
    assert moe.check_device_error(ws) == 0
    if repeat:
        y2 = moe.shared_forward(x, l1, l2, workspace=ws, act=act)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "not deterministic"
    kw = {} if situ is None else dict(activation="situ", beta=situ[0], linear_beta=situ[1])
    tok = None if tokens is None else np.asarray(tokens, np.int32)
    ref = oracle.shared_forward(bits(x), bits(l1), bits(l2), tokens=tok, **kw)["y"]
    got = y if tokens is None else y[torch.as_tensor(tok, device="cuda", dtype=torch.int64)]
    return compare_rows(got, ref, f"shared T={T} SH={SH} SI={SI}")


@pytest.mark.parametrize("T,SH,SI,seed", [
    (1, 256, 128, 1),        # one token
    (37, 512, 256, 2),       # ragged 32-token blocks
    (64, 512, 256, 27),      # 32-token blocks at the largest such T
    (100, 384, 256, 28),     # two 64-token blocks (64, 36 rows), odd output-tile count
    (300, 384, 256, 3),      # odd output-tile count: GEMM2's last pair holds one tile
    (1100, 256, 128, 4),     # 128-token blocks, ragged last block
    (128, 256, 256, 8),      # 64-token blocks at the largest such T
    (5, 128, 128, 24),       # the smallest shapes: one intermediate tile, one output tile (GEMM2 pair half empty)
])
def test_shared_small(moe, T, SH, SI, seed):
    run_and_compare(moe, T, SH, SI, seed)


def test_shared_situ(moe):
    run_and_compare(moe, 70, 256, 256, 5, situ=(1.25, 1.5))


def test_shared_situ_without_linear_term(moe):
    """SiTU with no linear_beta: the up projection enters unclipped, on the
    K-split cluster path (T = 8) and with 128-token blocks (T = 200)."""
    run_and_compare(moe, 8, 1024, 512, 25, situ=(2.0, None))
    run_and_compare(moe, 200, 512, 256, 26, situ=(0.75, None))


def test_shared_full_size_sampled(moe):
    """T = 8192 tokens, SH = 7168, SI = 2048, 8 sampled tokens (incl. the first
    and the last)."""
    T = 8192
    tokens = sorted(set(np.random.default_rng(6).choice(T, 6, replace=False).tolist()) | {0, T - 1})
    run_and_compare(moe, T, 7168, 2048, 6, tokens=tokens, repeat=False)


def test_shared_decode_size(moe):
    """T = 8 tokens (32-token blocks, most SMs idle), SH = 7168, SI = 2048."""
    run_and_compare(moe, 8, 7168, 2048, 7)


def test_shared_decode_size_situ(moe):
    """T = 8, full size, SiTU: the K-split path's last part runs the SiTU
    activation."""
    run_and_compare(moe, 8, 7168, 2048, 9, situ=(1.25, 1.5))


def test_shared_split_ragged_blocks(moe):
    """T = 40 at full size: two 32-token blocks (32 and 8 rows), each item's K
    cut into parts across a cluster."""
    run_and_compare(moe, 40, 7168, 2048, 10)


def test_shared_workspace_reuse(moe):
    """One zero-filled workspace through calls of different token counts
    (K-split and unsplit, both token-block sizes) and activations, then
    through a header as a call whose GEMM2 timed out leaves it (error word
    set, GEMM2's split counters at header words 192..319 nonzero): every
    result is bit-identical to a call on a fresh workspace, and the error word
    reports each call's own status."""
    SH, SI = 1024, 512
    ws = moe.shared_workspace(1100, SH, SI, "cuda")
    situ = moe.activation("situ", 1.25, 1.5)
    for T, act, seed in [(8, None, 11), (300, situ, 12), (8, situ, 13), (40, None, 14), (1100, None, 15),
                         (1, None, 16), (8, None, 11)]:
        x, l1, l2 = W.gen_shared(T, SH, SI, seed, "cuda")
        fresh = moe.shared_forward(x, l1, l2, workspace=moe.shared_workspace(T, SH, SI, "cuda"), act=act)
        got = moe.shared_forward(x, l1, l2, workspace=ws, act=act)
        assert moe.check_device_error(ws) == 0
        assert torch.equal(got.view(torch.int16), fresh.view(torch.int16)), f"T={T}"
    hdr = ws[:2048].view(torch.int32)
    hdr[0] = 2  # the timeout bit
    hdr[192:320] = 7
    x, l1, l2 = W.gen_shared(8, SH, SI, 17, "cuda")
    fresh = moe.shared_forward(x, l1, l2, workspace=moe.shared_workspace(8, SH, SI, "cuda"))
    got = moe.shared_forward(x, l1, l2, workspace=ws)
    assert moe.check_device_error(ws) == 0
    assert torch.equal(got.view(torch.int16), fresh.view(torch.int16))


@pytest.mark.parametrize("T,SH,SI,seed,situ", [
    (300, 1024, 512, 18, None),          # 128-token blocks (128, 128, 44 rows), both GEMMs K-split
    (600, 640, 384, 19, None),           # odd output-tile count, GEMM1 split in two
    (290, 512, 1024, 20, (1.25, 1.5)),   # SiTU on the 128-token split path
    (129, 1024, 512, 22, None),          # the smallest such T: a last block of one token
])
def test_shared_split_128_token_blocks(moe, T, SH, SI, seed, situ):
    """More than 128 tokens (128-token blocks) with fewer work items than SMs:
    each item's K is cut into parts whose fp32 partials (128 tokens per block)
    the item's last part adds in part order; every token checked."""
    run_and_compare(moe, T, SH, SI, seed, situ=situ)


def test_shared_split_128_full_size_sampled(moe):
    """T = 300 at SH = 7168, SI = 2048 (GEMM1 split three ways over 48 items),
    16 sampled tokens from every block, the last included."""
    T = 300
    tokens = sorted(set(np.random.default_rng(21).choice(T, 13, replace=False).tolist()) | {0, 255, T - 1})
    run_and_compare(moe, T, 7168, 2048, 21, tokens=tokens)


def test_shared_split_global_partials(moe):
    """An item cut into more K parts than a thread-block cluster holds (T = 8,
    SH = 7168, SI = 128: one GEMM1 item in 28 parts) adds its partials through
    global memory, the last part to finish reducing them."""
    run_and_compare(moe, 8, 7168, 128, 23)


@pytest.mark.parametrize("T,SH,SI,seed,situ", [
    (96, 1024, 512, 29, None),           # 64-token blocks (64, 32 rows), both GEMMs K-split
    (65, 768, 384, 30, (1.25, 1.5)),     # the smallest such T: a last block of one token, SiTU
])
def test_shared_split_64_token_blocks(moe, T, SH, SI, seed, situ):
    """65 to 128 tokens: 64-token blocks, each item's K cut into parts; every
    token checked."""
    run_and_compare(moe, T, SH, SI, seed, situ=situ)


def test_shared_64_token_blocks_full_size(moe):
    """T = 96 at SH = 7168, SI = 2048 (two 64-token blocks, 32 GEMM1 items
    split four ways), every token."""
    run_and_compare(moe, 96, 7168, 2048, 31)
