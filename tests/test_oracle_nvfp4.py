"""Pins for the oracle's NVFP4 variant (the "NVFP4 Mega MoE Kernel -- Mojo
Rewrite" README: E2M1 values, one UE4M3 scale per 16 K elements, activations
quantised to FP4 as well).

UE4M3 decoding is pinned to torch's float8_e4m3fn; the scale rule (smallest
UE4M3 value s with 6*s >= amax) to numpy's searchsorted over the sorted
codebook; the codes to a brute-force nearest-E2M1 search (ties to the even
mantissa) of the fp32 quotient; the layer to a float64 numpy evaluation with
its own decoders, plus the same invariants as the FP8 x FP4 layer.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

OCP_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
UE4M3 = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()  # codes 0..126


def test_ue4m3_codebook_matches_torch():
    for c in range(127):
        assert oracle.ue4m3_value(c) == UE4M3[c]
    assert np.isnan(oracle.ue4m3_value(0x7F))
    assert oracle.ue4m3_value(0x80 | 0x38) == 1.0     # the sign bit is not part of a UE4M3 scale


def expected_scale(amax):
    if amax == 0.0:
        return 0x38
    i = int(np.searchsorted(6.0 * UE4M3[1:], amax, side="left")) + 1  # first code with 6*s >= amax
    return min(i, 0x7E)


def test_scale_rule_against_searchsorted():
    rng = np.random.default_rng(7)
    amaxes = list(10.0 ** rng.uniform(-4, 3.5, 4000))
    for c in range(1, 127):                   # exact boundaries and their neighbours
        b = 6.0 * UE4M3[c]
        amaxes += [b, np.nextafter(b, 0.0), np.nextafter(b, np.inf)]
    amaxes += [0.0, 1e-9, 6 * 448.0, 6 * 448.0 * 1.5]
    for a in amaxes:
        assert oracle.nvfp4_scale(float(a)) == expected_scale(float(a)), a
    assert UE4M3[oracle.nvfp4_scale(1.0)] == 0.171875     # worked by hand: smallest E4M3 >= 1/6


def brute_e2m1(q):
    """nearest E2M1 code of each fp32 value, ties to the even mantissa, sign kept"""
    out = np.empty(q.shape, np.uint8)
    for i, v in np.ndenumerate(q):
        a = abs(float(v))
        d = np.abs(OCP_E2M1 - a)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (8 if np.signbit(v) else 0)
    return out


def test_quantize_codes_brute_force():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((24, 64)) * np.exp(rng.uniform(-6, 3, (24, 1)))).astype(np.float32)
    x[3] = 0.0
    x[4, :16] = -1e-30
    packed, sf = oracle.quantize_nvfp4(x)
    for r in range(x.shape[0]):
        for g in range(x.shape[1] // 16):
            blk = x[r, g * 16:(g + 1) * 16]
            c = expected_scale(float(np.abs(blk.astype(np.float64)).max()))
            assert sf[r, g] == c
            q = (blk / np.float32(UE4M3[c])).astype(np.float32)   # the fp32 quotient
            codes = brute_e2m1(q)
            got = np.stack([packed[r, g * 8:(g + 1) * 8] & 0xF, packed[r, g * 8:(g + 1) * 8] >> 4], -1).ravel()
            assert np.array_equal(got, codes), (r, g)


def test_representable_values_round_trip():
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, (8, 32))
    scale_codes = rng.integers(20, 90, (8, 2))
    v = np.where(codes & 8, -1.0, 1.0) * OCP_E2M1[codes & 7] * np.repeat(UE4M3[scale_codes], 16, axis=1)
    v[:, 0] = 6.0 * UE4M3[scale_codes[:, 0]]    # each group's amax is 6 * its scale
    v[:, 16] = 6.0 * UE4M3[scale_codes[:, 1]]
    packed, sf = oracle.quantize_nvfp4(v.astype(np.float32))
    assert np.array_equal(sf, scale_codes)
    back = dq(packed, sf)
    assert np.array_equal(back, v)


def dq(packed, sf):
    lo, hi = packed & 0xF, packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)
    v = np.where(codes & 8, -1.0, 1.0) * OCP_E2M1[codes & 7]
    return v * np.repeat(UE4M3[sf], 16, axis=-1)


def make(w, routing=None):
    x = W.gen_x(w).float().numpy()
    idx, tw = routing if routing is not None else W.gen_routing(w)
    l1 = {e: W.gen_l1(w, e).float().numpy() for e in range(w.E)}
    l2 = {e: W.gen_l2(w, e).float().numpy() for e in range(w.E)}
    xq, xs, ex = oracle.quantize_inputs(x, l1, l2, fmt="nvfp4")
    return xq, xs, idx.numpy(), tw.numpy(), ex


SMALL = [W.custom("n1", T=6, E=4, k=2, H=64, I=64, seed=61), W.custom("n2", T=5, E=3, k=3, H=96, I=32, seed=62)]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_nvfp4_layer_matches_float64_brute_force(w):
    xq, xs, idx, tw, ex = make(w)
    r = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, intermediates=True, fmt="nvfp4")
    xd = dq(xq, xs)
    for t in range(w.T):
        out = np.zeros(w.H)
        for j in range(w.k):
            e = int(idx[t, j])
            c1 = dq(ex[e][0], ex[e][1]) @ xd[t]
            g, u = c1[:w.I], c1[w.I:]
            h = g / (1.0 + np.exp(-g)) * u
            np.testing.assert_allclose(r["h_pre"][t, j], h, rtol=1e-5, atol=1e-6)
            # the requant: scale rule and codes of the oracle's own pre-requant h
            hp = r["h_pre"][t, j].astype(np.float32)
            for gi in range(w.I // 16):
                blk = hp[gi * 16:(gi + 1) * 16]
                c = expected_scale(float(np.abs(blk.astype(np.float64)).max()))
                assert r["h_sf"][t, j, gi] == c
                codes = brute_e2m1((blk / np.float32(UE4M3[c])).astype(np.float32))
                hb = r["h_q"][t, j, gi * 8:(gi + 1) * 8]
                assert np.array_equal(np.stack([hb & 0xF, hb >> 4], -1).ravel(), codes)
            hd = dq(r["h_q"][t, j][None], r["h_sf"][t, j][None])[0]
            y = dq(ex[e][2], ex[e][3]) @ hd
            out += float(tw[t, j]) * y
        np.testing.assert_allclose(r["out_f32"][t], out, rtol=2e-5, atol=2e-5 * np.abs(out).max())


def test_nvfp4_layer_permutation_and_identical_experts():
    w = W.custom("n3", T=8, E=3, k=2, H=64, I=64, seed=63)
    xq, xs, idx, tw, ex = make(w)
    r = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, fmt="nvfp4")
    perm = np.random.default_rng(1).permutation(w.T)
    rp = oracle.forward(xq[perm], xs[perm], idx[perm], tw[perm], ex, w.E, w.H, w.I, fmt="nvfp4")
    assert np.array_equal(rp["out_bf16"], r["out_bf16"][perm])
    same = {e: ex[0] for e in range(w.E)}
    ones = np.ones_like(tw)
    rs = oracle.forward(xq, xs, idx, ones, same, w.E, w.H, w.I, fmt="nvfp4")
    r1 = oracle.forward(xq, xs, idx[:, :1], ones[:, :1], same, w.E, w.H, w.I, fmt="nvfp4")
    f = oracle.bf16_bits_to_f32(r1["out_bf16"]).astype(np.float64)
    got = oracle.bf16_bits_to_f32(rs["out_bf16"]).astype(np.float64)
    np.testing.assert_allclose(got, w.k * f, rtol=2 ** -7, atol=1e-6)
