"""Weight layout A/B (the DeepGEMM PR #394 Correctness section compares the
row-major and packet layouts for bitwise-identical outputs): the row-major
layout (FP4 bodies read in place, scale blocks in a separate array) must give
exactly the packet layout's output, and its scale blocks must be exactly the
ones inside the packets."""
import gc

import numpy as np
import pytest
import torch

import workloads as W
from cases import compare_rows, experts_of, gpu_layer, oracle_side
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


@pytest.mark.parametrize("E,H,I", [(2, 256, 128), (3, 384, 256), (2, 384, 384)])
def test_scale_blocks_equal_the_packets(moe, E, H, I):
    g = torch.Generator(device="cuda").manual_seed(E * 1000 + H + I)
    l1 = torch.randn((E, 2 * I, H), generator=g, device="cuda").to(torch.bfloat16)
    l2 = torch.randn((E, H, I), generator=g, device="cuda").to(torch.bfloat16)
    a, b = moe.quantize_fp4(l1.view(E * 2 * I, H))
    c, d = moe.quantize_fp4(l2.view(E * H, I))
    a, b = a.view(E, 2 * I, H // 2), b.view(E, 2 * I, H // 32)
    c, d = c.view(E, H, I // 2), d.view(E, H, I // 32)
    p1, p2 = moe.transform_weights(a, b, c, d)
    s1, s2 = moe.transform_scales(b, d)
    for pk, sc in ((p1, s1), (p2, s2)):
        n = sc.numel() // 512
        assert pk.numel() == n * 8704
        assert torch.equal(pk.view(n, 8704)[:, 8192:], sc.view(n, 512))


CASES = [
    W.WORKLOADS[0],                                                          # 160-row chunks
    W.custom("ragged_odd_tiles", T=37, E=5, k=3, H=384, I=256, seed=21),     # H/128 odd: padded pair
    W.custom("small_chunks", T=6, E=64, k=2, H=384, I=256, seed=51),         # 32-row chunks, odd H tiles
    W.custom("multichunk", T=300, E=2, k=2, H=256, I=128, seed=22),
    W.custom("max_I", T=20, E=2, k=2, H=256, I=8192, seed=44),
]


def run_both(moe, w, routing=None, act=None):
    g = gpu_layer(w, routing=routing, rowmajor=True)
    ws = torch.empty(moe.workspace_bytes(w.T, w.E, w.k, w.H, w.I), dtype=torch.uint8, device="cuda")
    a = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I, workspace=ws, act=act)
    assert moe.check_device_error(ws) == 0
    b = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], None, None, w.E, w.H, w.I, workspace=ws, act=act,
                    weights=g["rm"])
    assert moe.check_device_error(ws) == 0
    return g, a, b


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_row_major_output_is_bitwise_the_packets(moe, w):
    g, a, b = run_both(moe, w)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    if w.name == "ragged_odd_tiles":
        # and against the oracle, every token
        idx = g["idx"].cpu().numpy()
        tok = np.arange(w.T)
        xq, xs, ex = oracle_side(w, g["x"], g["idx"], experts_of(idx, tok, w.E))
        ref = oracle.forward(xq, xs, idx, g["tw"].cpu().numpy(), ex, w.E, w.H, w.I)
        compare_rows(b, ref["out_bf16"], w.name)


def test_row_major_situ_bitwise(moe):
    _, a, b = run_both(moe, W.custom("situ_layouts", T=40, E=6, k=2, H=256, I=256, seed=52),
                       act=moe.activation("situ", 1.25, 1.5))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("cfg", [1, 3])
def test_row_major_full_size_bitwise(moe, cfg):
    """Decode (32-row chunks) and prefill (160-row chunks) at full size."""
    w = W.WORKLOADS[cfg]
    _, a, b = run_both(moe, w, routing=W.gen_routing(w, "cuda"))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    del a, b
    gc.collect()
    torch.cuda.empty_cache()
