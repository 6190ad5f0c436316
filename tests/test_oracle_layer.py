"""Pins for the oracle's layer arithmetic.

The reference here is a float64 numpy evaluation of every selected expert of
every token, written from the definition (dequantise, dense matmul, SwiGLU with
the gate first, GEMM2, weighted sum over the k slots) with its own decoders
(torch's float8 view for E4M3, the OCP table for E2M1, ldexp for UE8M0).  The
FP8 requantisation of the SwiGLU output is the one step both share: the
reference takes the oracle's h codes as GEMM2's input, after checking them
against torch's RNE cast of the oracle's pre-requant h.  Invariants: the
single-expert dense special case, token-permutation equivariance, identical
experts with unit weights summing to k*f(x), determinism across thread counts.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

OCP_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def dq_e4m3(codes, sf):
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    s = np.ldexp(1.0, sf.astype(np.int64) - 127)
    return v * np.repeat(s, 32, axis=-1)


def dq_e2m1(packed, sf):
    lo, hi = packed & 0xF, packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)
    v = np.where(codes & 8, -1.0, 1.0) * OCP_E2M1[codes & 7]
    return v * np.repeat(np.ldexp(1.0, sf.astype(np.int64) - 127), 32, axis=-1)


def make(w: W.Workload, routing=None):
    x = W.gen_x(w).float().numpy()
    idx, tw = routing if routing is not None else W.gen_routing(w)
    l1 = {e: W.gen_l1(w, e).float().numpy() for e in range(w.E)}
    l2 = {e: W.gen_l2(w, e).float().numpy() for e in range(w.E)}
    xq, xs, ex = oracle.quantize_inputs(x, l1, l2)
    return xq, xs, idx.numpy(), tw.numpy(), ex


def brute_force(xq, xs, idx, tw, ex, I, h_codes=None, h_sf=None):
    """float64 evaluation; GEMM2 input = given h codes (else requantised by torch)."""
    T, k = idx.shape
    xd = dq_e4m3(xq, xs)
    hs, ys, outs = [], [], []
    for t in range(T):
        out = np.zeros(xq.shape[1])
        hrow, yrow = [], []
        for j in range(k):
            e = int(idx[t, j])
            w1 = dq_e2m1(ex[e][0], ex[e][1])
            w2 = dq_e2m1(ex[e][2], ex[e][3])
            c1 = w1 @ xd[t]
            g, u = c1[:I], c1[I:]
            h = g / (1.0 + np.exp(-g)) * u
            hrow.append(h)
            hd = dq_e4m3(h_codes[t, j], h_sf[t, j])
            y = w2 @ hd
            yrow.append(y)
            out += float(tw[t, j]) * y
        hs.append(hrow)
        ys.append(yrow)
        outs.append(out)
    return np.array(hs), np.array(ys), np.array(outs)


SMALL = [W.custom("t1", T=6, E=4, k=2, H=64, I=64, seed=11),
         W.custom("t2", T=5, E=3, k=3, H=96, I=32, seed=12),
         W.WORKLOADS[0]]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_layer_matches_float64_brute_force(w):
    xq, xs, idx, tw, ex = make(w)
    r = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, intermediates=True)
    h, y, out = brute_force(xq, xs, idx, tw, ex, w.I, r["h_q"], r["h_sf"])
    # GEMM1 + SwiGLU before requantisation: fp32 accumulation vs float64
    hmax = np.abs(h).max()
    assert np.abs(r["h_pre"] - h).max() <= 1e-5 * hmax
    # the requantised codes are torch's RNE cast of the oracle's own h with the
    # exact scale rule
    hp = r["h_pre"].reshape(-1, w.I // 32, 32).astype(np.float64)
    amax = np.abs(hp).max(-1)
    e = np.where(amax > 0, np.ceil(np.log2(np.where(amax > 0, amax, 1) / 448.0)), 0)
    # log2 may land exactly on an integer boundary: fix up with exact comparisons
    e = e + (amax > 448.0 * np.ldexp(1.0, e.astype(int))) - (amax <= 448.0 * np.ldexp(1.0, e.astype(int) - 1)) * (amax > 0)
    assert np.array_equal(r["h_sf"].reshape(-1, w.I // 32), (e + 127).astype(np.uint8))
    q = torch.from_numpy((hp / np.ldexp(1.0, e.astype(int))[..., None]).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q.view(torch.uint8).numpy().reshape(r["h_q"].shape), r["h_q"])
    # GEMM2 and the combine
    assert np.abs(r["y"] - y).max() <= 1e-5 * np.abs(y).max()
    assert np.abs(r["out_f32"] - out).max() <= 1e-5 * np.abs(out).max()
    ref_bf16 = torch.from_numpy(r["out_f32"]).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(r["out_bf16"], ref_bf16)


def test_double_mode_bounds_fp32_rounding():
    w = SMALL[0]
    xq, xs, idx, tw, ex = make(w)
    rd = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, precision="double", intermediates=True)
    _, _, out = brute_force(xq, xs, idx, tw, ex, w.I, rd["h_q"], rd["h_sf"])
    assert np.abs(rd["out_f32"] - out).max() <= 1e-6 * np.abs(out).max()
    rf = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I)
    a, b = oracle.bf16_bits_to_f32(rf["out_bf16"]), oracle.bf16_bits_to_f32(rd["out_bf16"])
    rel = np.linalg.norm(a - b, axis=1) / np.linalg.norm(b, axis=1)
    assert rel.max() < 1e-2


def test_single_expert_is_dense_quantised_ffn():
    w = W.custom("dense", T=7, E=1, k=1, H=64, I=96, seed=13)
    idx = np.zeros((7, 1), np.int64)
    xq, xs, _, _, ex = make(w, routing=(torch.zeros(7, 1, dtype=torch.int64), torch.ones(7, 1)))
    r = oracle.forward(xq, xs, idx, np.ones((7, 1), np.float32), ex, 1, w.H, w.I, intermediates=True)
    xd = dq_e4m3(xq, xs)
    w1 = dq_e2m1(ex[0][0], ex[0][1])
    w2 = dq_e2m1(ex[0][2], ex[0][3])
    c1 = xd @ w1.T
    h = c1[:, : w.I] / (1 + np.exp(-c1[:, : w.I])) * c1[:, w.I:]
    assert np.abs(r["h_pre"][:, 0] - h).max() <= 1e-5 * np.abs(h).max()
    dense = dq_e4m3(r["h_q"][:, 0], r["h_sf"][:, 0]) @ w2.T
    assert np.abs(r["out_f32"] - dense).max() <= 1e-5 * np.abs(dense).max()


def test_token_permutation_equivariance_is_bitwise():
    w = W.WORKLOADS[0]
    xq, xs, idx, tw, ex = make(w)
    p = np.random.default_rng(7).permutation(w.T)
    a = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I)["out_bf16"]
    b = oracle.forward(xq[p], xs[p], idx[p], tw[p], ex, w.E, w.H, w.I)["out_bf16"]
    assert np.array_equal(a[p], b)


@pytest.mark.parametrize("k", [2, 3, 4])
def test_identical_experts_unit_weights_sum_to_k_f(k):
    w = W.custom("same", T=9, E=5, k=k, H=64, I=64, seed=14)
    xq, xs, idx, _, ex = make(w)
    same = {e: ex[0] for e in range(w.E)}
    ones = np.ones((w.T, k), np.float32)
    out = oracle.forward(xq, xs, idx, ones, same, w.E, w.H, w.I)["out_bf16"]
    f = oracle.forward(xq, xs, np.zeros((w.T, 1), np.int64), np.ones((w.T, 1), np.float32),
                       {0: ex[0]}, 1, w.H, w.I)["out_f32"]
    ref = torch.from_numpy((k * f.astype(np.float64)).astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = out.view(np.int16)
    # within one bf16 ulp (same sign, so the bit patterns differ by <= 1)
    assert np.abs(got.astype(np.int32) - ref.astype(np.int32)).max() <= 1


def test_deterministic_across_thread_counts_and_token_subsets():
    w = W.WORKLOADS[0]
    xq, xs, idx, tw, ex = make(w)
    a = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, threads=1)["out_bf16"]
    b = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, threads=0)["out_bf16"]
    assert np.array_equal(a, b)
    sel = np.array([63, 0, 17], np.int32)
    c = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, tokens=sel)["out_bf16"]
    assert np.array_equal(c, a[sel])


def test_dropped_slot_contributes_nothing():
    w = W.custom("drop", T=4, E=3, k=2, H=64, I=64, seed=15)
    xq, xs, idx, tw, ex = make(w)
    bad = idx.copy()
    bad[1, 1] = 7
    r = oracle.forward(xq, xs, bad, tw, ex, w.E, w.H, w.I, intermediates=True)
    only = oracle.forward(xq[1:2], xs[1:2], idx[1:2, :1], tw[1:2, :1], ex, w.E, w.H, w.I)
    assert np.array_equal(r["out_bf16"][1], only["out_bf16"][0])


def test_missing_expert_weights_raise():
    w = SMALL[0]
    xq, xs, idx, tw, ex = make(w)
    partial = {e: ex[e] for e in list(ex)[:1]}
    with pytest.raises(KeyError):
        oracle.forward(xq, xs, idx, tw, partial, w.E, w.H, w.I)


# ---------------------------------------------------------------- SiTU
def situ64(g, u, beta, linear_beta):
    """SiTU in float64: sigmoid(g) * beta*tanh(g/beta) * beta_lin*tanh(u/beta_lin)
    (up factor u when beta_lin is absent)."""
    up = u if linear_beta is None else linear_beta * np.tanh(u / linear_beta)
    return 1.0 / (1.0 + np.exp(-g)) * (beta * np.tanh(g / beta)) * up


@pytest.mark.parametrize("beta,linear_beta", [(1.25, 1.5), (0.5, None), (3.0, 0.25)])
def test_situ_matches_float64_brute_force(beta, linear_beta):
    w = W.custom("situ", T=6, E=4, k=2, H=64, I=64, seed=16)
    xq, xs, idx, tw, ex = make(w)
    r = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, intermediates=True,
                       activation="situ", beta=beta, linear_beta=linear_beta)
    xd = dq_e4m3(xq, xs)
    for t in range(w.T):
        out = np.zeros(w.H)
        for j in range(w.k):
            e = int(idx[t, j])
            c1 = dq_e2m1(ex[e][0], ex[e][1]) @ xd[t]
            h = situ64(c1[: w.I], c1[w.I:], beta, linear_beta)
            assert np.abs(r["h_pre"][t, j] - h).max() <= 1e-5 * max(np.abs(h).max(), 1e-30)
            y = dq_e2m1(ex[e][2], ex[e][3]) @ dq_e4m3(r["h_q"][t, j], r["h_sf"][t, j])
            out += float(tw[t, j]) * y
        assert np.abs(r["out_f32"][t] - out).max() <= 1e-5 * np.abs(out).max()


def test_situ_with_large_betas_is_swiglu():
    w = W.custom("situ_lim", T=5, E=3, k=2, H=64, I=96, seed=17)
    xq, xs, idx, tw, ex = make(w)
    a = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, intermediates=True, precision="double",
                       activation="situ", beta=1e9, linear_beta=1e9)
    b = oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, intermediates=True, precision="double")
    assert np.abs(a["h_pre"] - b["h_pre"]).max() <= 1e-6 * np.abs(b["h_pre"]).max()


def test_situ_rejects_bad_coefficients():
    w = W.custom("situ_bad", T=2, E=2, k=1, H=32, I=32, seed=18)
    xq, xs, idx, tw, ex = make(w)
    for beta, lb in ((0.0, 1.0), (-1.0, None), (float("inf"), None), (1.0, float("nan"))):
        with pytest.raises(ValueError):
            oracle.forward(xq, xs, idx, tw, ex, w.E, w.H, w.I, activation="situ", beta=beta, linear_beta=lb)
