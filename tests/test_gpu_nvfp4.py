"""GPU parity of the NVFP4 variant (the "NVFP4 Mega MoE Kernel -- Mojo Rewrite"
README: E2M1 values with UE4M3 per-16 scales for activations, weights and the
intermediate, tcgen05 kind::mxf4nvf4 with scale_vec::4X) against the oracle's
NVFP4 path: quantiser codes and scales bit-exact, packets checked against their
sources, the layer per token row within the layer's tolerance."""
import gc

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from cases import compare_rows, experts_of, gpu_layer_nvfp4, oracle_side_nvfp4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def test_quantize_nvfp4_bit_exact(moe):
    g = torch.Generator(device="cuda").manual_seed(71)
    x = (torch.randn((64, 512), generator=g, device="cuda") *
         torch.exp(torch.empty((64, 1), device="cuda").uniform_(-9, 4, generator=g))).to(torch.bfloat16)
    x[0] = 0.0
    x[1, :16] = -1e-30
    x[2, :] = 3000.0 * torch.sign(x[2, :])   # amax above 6 * 448: the largest scale, saturated codes
    x[3, 16:32] = torch.tensor([6.0 * 0.171875] + [0.0] * 15, device="cuda")  # amax = 6 * s exactly
    q, sf = moe.quantize_nvfp4(x)
    oq, osf = oracle.quantize_nvfp4(x.float().cpu().numpy())
    assert np.array_equal(sf.cpu().numpy(), osf)
    assert np.array_equal(q.cpu().numpy(), oq)


def test_nvfp4_packets_hold_their_sources(moe):
    E, H, I = 2, 512, 256
    g = torch.Generator(device="cuda").manual_seed(72)
    l1 = torch.randn((E * 2 * I, H), generator=g, device="cuda").to(torch.bfloat16)
    l2 = torch.randn((E * H, I), generator=g, device="cuda").to(torch.bfloat16)
    a, b = moe.quantize_nvfp4(l1)
    c, d = moe.quantize_nvfp4(l2)
    a, b, c, d = a.view(E, 2 * I, H // 2), b.view(E, 2 * I, H // 16), c.view(E, H, I // 2), d.view(E, H, I // 16)
    p1, p2 = moe.transform_weights_nvfp4(a, b, c, d)
    P = 18432
    p1, p2 = p1.view(-1, P).cpu().numpy(), p2.view(-1, P).cpu().numpy()
    a, b, c, d = a.cpu().numpy(), b.cpu().numpy(), c.cpu().numpy(), d.cpu().numpy()
    r = np.arange(128)
    img_off = (r % 32) * 16 + (r // 32) * 4          # byte of (row r, group 0) in a 512-byte image

    def check(pk, body, sfs, rows):
        assert np.array_equal(pk[:16384].reshape(128, 128), body[rows])
        for s in range(4):
            im = pk[16384 + 512 * s:16384 + 512 * (s + 1)]
            for gi in range(4):
                assert np.array_equal(im[img_off + gi], sfs[rows, 4 * s + gi])
    # L1 packet ((e * (I/128) + it) * (H/256) + kb) * 2 + slot: slot 0 gate rows, 1 up rows
    KB1 = H // 256
    for e, it, kb, slot in [(0, 0, 0, 0), (1, 1, 1, 1), (0, 1, 0, 1)]:
        pk = p1[((e * (I // 128) + it) * KB1 + kb) * 2 + slot]
        rows = slot * I + it * 128 + r
        check(pk, a[e][:, kb * 128:(kb + 1) * 128], b[e][:, kb * 16:(kb + 1) * 16], rows)
    # L2 packet ((e * (H/256) + p) * (I/256) + kb) * 2 + slot: tile 2p + slot
    KB2 = I // 256
    for e, pp, kb, slot in [(0, 0, 0, 1), (1, 1, 0, 0)]:
        pk = p2[((e * (H // 256) + pp) * KB2 + kb) * 2 + slot]
        rows = (2 * pp + slot) * 128 + r
        check(pk, c[e][:, kb * 128:(kb + 1) * 128], d[e][:, kb * 16:(kb + 1) * 16], rows)


def run_and_compare_nv(moe, w, routing=None, tokens=None, situ=None, check_repeat=True):
    g = gpu_layer_nvfp4(w, routing=routing)
    ws = torch.empty(moe.workspace_bytes(w.T, w.E, w.k, w.H, w.I), dtype=torch.uint8, device="cuda")
    act = None if situ is None else moe.activation("situ", situ[0], situ[1])
    out = moe.forward_nvfp4(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I,
                            workspace=ws, act=act)
    status = moe.check_device_error(ws)
    if check_repeat:
        out2 = moe.forward_nvfp4(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I,
                                 workspace=ws, act=act)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "not deterministic"
    idx = g["idx"].cpu().numpy()
    tok = np.arange(w.T) if tokens is None else np.asarray(tokens)
    xq, xs, ex = oracle_side_nvfp4(w, g["x"], experts_of(idx, tok, w.E))
    assert np.array_equal(g["xq"].cpu().numpy(), xq) and np.array_equal(g["xs"].cpu().numpy(), xs)
    kw = {} if situ is None else dict(activation="situ", beta=situ[0], linear_beta=situ[1])
    ref = oracle.forward(xq, xs, idx, g["tw"].cpu().numpy(), ex, w.E, w.H, w.I, fmt="nvfp4",
                         tokens=None if tokens is None else tok.astype(np.int32), **kw)
    compare_rows(out[torch.as_tensor(tok, device="cuda")], ref["out_bf16"], w.name)
    del g, ws, out
    gc.collect()
    torch.cuda.empty_cache()
    return status


SMALL = [
    W.WORKLOADS[0],                                                       # 160-row chunks
    W.custom("nv_small_chunks", T=6, E=64, k=2, H=512, I=256, seed=81),   # 32-row chunks
    W.custom("nv_ragged", T=37, E=5, k=3, H=512, I=256, seed=82),
    W.custom("nv_multichunk", T=300, E=2, k=2, H=256, I=512, seed=83),
    W.custom("nv_one_token", T=1, E=16, k=4, H=512, I=256, seed=84),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_nvfp4_layer_small(moe, w):
    assert run_and_compare_nv(moe, w) == 0


def test_nvfp4_layer_split_units(moe):
    """One chunk: every item of both GEMMs is cut along K into units whose
    partial accumulators the last unit adds (GEMM2 with three 256-K stages)."""
    from test_gpu_layer import one_expert_routing, split_of
    w = W.custom("nv_split", T=32, E=64, k=1, H=1024, I=768, seed=86)
    idx, tw = one_expert_routing(w, [7])
    ic = idx.numpy()
    assert split_of(ic, w, True, mx=False) >= 2 and split_of(ic, w, False, mx=False) >= 2
    assert run_and_compare_nv(moe, w, routing=(idx, tw)) == 0


def test_nvfp4_layer_side_list(moe):
    """NVFP4 with both chunk lists (160-row main chunks, 32-row side chunks)."""
    from test_gpu_layer import SIDE_COUNTS, side_list_routing
    w = W.custom("nv_side_list", T=100, E=8, k=2, H=512, I=256, seed=87)
    assert run_and_compare_nv(moe, w, routing=side_list_routing(w, SIDE_COUNTS, 87)) == 0


def test_nvfp4_layer_situ(moe):
    assert run_and_compare_nv(moe, W.custom("nv_situ", T=40, E=6, k=2, H=256, I=256, seed=85), situ=(1.25, 1.5)) == 0


def test_nvfp4_layer_decode_full(moe):
    assert run_and_compare_nv(moe, W.WORKLOADS[1]) == 0


def test_nvfp4_layer_prefill_sampled(moe):
    w = W.WORKLOADS[3]
    idx, tw = W.gen_routing(w, "cuda")
    tokens = sorted(set(np.random.default_rng(9).choice(w.T, 6, replace=False).tolist()) | {0, w.T - 1})
    assert run_and_compare_nv(moe, w, routing=(idx, tw), tokens=tokens, check_repeat=False) == 0
