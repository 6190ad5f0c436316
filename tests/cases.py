"""Shared helpers of the GPU parity tests: build a layer's inputs for the CUDA
library (quantised and transformed by the library itself) and, separately,
for the oracle (quantised by the oracle from the same bf16 draws)."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import workloads as W

# Per-token-row tolerances of the layer output against the oracle.
REL_L2_TOL = 1e-2
MAX_ABS_TOL = 5e-2   # times max |row| of the oracle output


def gpu_layer(w: W.Workload, routing=None, gen_device="cuda", device="cuda", rowmajor=False):
    """Inputs of the CUDA path: bf16 draws quantised and transformed by the library.
    With rowmajor, also the same weights in the row-major layout ("rm")."""
    import moe_expert_layer_08_b200 as moe
    x = W.gen_x(w, gen_device).to(device)
    if routing is None:
        routing = W.gen_routing(w, gen_device)
    idx, tw = routing[0].to(device).contiguous(), routing[1].to(device).contiguous()
    xq, xs = moe.quantize_fp8(x)
    n1, n2 = moe.transformed_weight_bytes(w.E, w.H, w.I)
    l1_t = torch.empty(n1, dtype=torch.uint8, device=device)
    l2_t = torch.empty(n2, dtype=torch.uint8, device=device)
    p1, p2 = n1 // w.E, n2 // w.E
    if rowmajor:
        u8 = dict(dtype=torch.uint8, device=device)
        r1 = torch.empty((w.E, 2 * w.I, w.H // 2), **u8)
        r2 = torch.empty((w.E, w.H, w.I // 2), **u8)
        s1 = torch.empty((w.E, 2 * w.I, w.H // 32), **u8)
        s2 = torch.empty((w.E, w.H, w.I // 32), **u8)
        m1, m2 = moe.transformed_scale_bytes(w.E, w.H, w.I)
        s1_t = torch.empty(m1, **u8)
        s2_t = torch.empty(m2, **u8)
        q1, q2 = m1 // w.E, m2 // w.E
    for e in range(w.E):
        a, b = moe.quantize_fp4(W.gen_l1(w, e, gen_device).to(device))
        c, d = moe.quantize_fp4(W.gen_l2(w, e, gen_device).to(device))
        moe.transform_weights(a[None], b[None], c[None], d[None],
                              out=(l1_t[e * p1:(e + 1) * p1], l2_t[e * p2:(e + 1) * p2]))
        if rowmajor:
            r1[e], s1[e], r2[e], s2[e] = a, b, c, d
            moe.transform_scales(b[None], d[None], out=(s1_t[e * q1:(e + 1) * q1], s2_t[e * q2:(e + 1) * q2]))
    g = dict(x=x, xq=xq, xs=xs, idx=idx, tw=tw, l1_t=l1_t, l2_t=l2_t)
    if rowmajor:
        g["rm"] = moe.RowMajorWeights(r1, s1_t, r2, s2_t)
    return g


def oracle_side(w: W.Workload, x_bf16: torch.Tensor, idx: torch.Tensor, experts, gen_device="cuda"):
    """Oracle inputs from the same bf16 draws: x and the listed experts'
    weights quantised by the oracle (in a thread pool: the C code releases the GIL)."""
    xq, xs = oracle.quantize_e4m3(x_bf16.float().cpu().numpy())
    experts = sorted(set(int(e) for e in experts))

    def quant(item):
        e, l1, l2 = item
        a, b = oracle.quantize_e2m1(l1)
        c, d = oracle.quantize_e2m1(l2)
        return e, (a, b, c, d)

    out = {}
    workers = max(1, min(len(experts), os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as pool:
        futs = []
        for e in experts:
            l1 = W.gen_l1(w, e, gen_device).float().cpu().numpy()
            l2 = W.gen_l2(w, e, gen_device).float().cpu().numpy()
            futs.append(pool.submit(quant, (e, l1, l2)))
        for f in futs:
            e, mats = f.result()
            out[e] = mats
    return xq, xs, out


def experts_of(idx: np.ndarray, tokens, E: int):
    sel = idx[np.asarray(tokens)].ravel()
    return sorted(set(int(e) for e in sel if 0 <= e < E))


def compare_rows(got: torch.Tensor, ref_bits: np.ndarray, what: str = ""):
    """Per token row: rel L2 <= REL_L2_TOL and max abs <= MAX_ABS_TOL * max |row|."""
    g = got.float().cpu().numpy().astype(np.float64)
    r = oracle.bf16_bits_to_f32(ref_bits).astype(np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    diff = g - r
    rn = np.linalg.norm(r, axis=1)
    zero = rn == 0
    assert np.all(g[zero] == 0), f"{what}: rows whose reference is zero are not zero"
    rel = np.linalg.norm(diff, axis=1)[~zero] / rn[~zero]
    mabs = np.abs(diff).max(axis=1)[~zero] / np.abs(r).max(axis=1)[~zero]
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= REL_L2_TOL, f"{what}: worst row rel L2 {worst:.3e}"
    assert (float(mabs.max()) if mabs.size else 0.0) <= MAX_ABS_TOL, f"{what}: max abs {mabs.max():.3e}"
    return worst


def gpu_layer_nvfp4(w: W.Workload, routing=None, gen_device="cuda", device="cuda"):
    """NVFP4 inputs of the CUDA path: the same bf16 draws quantised to E2M1 +
    UE4M3 per 16 and packed by the library."""
    import moe_expert_layer_08_b200 as moe
    x = W.gen_x(w, gen_device).to(device)
    if routing is None:
        routing = W.gen_routing(w, gen_device)
    idx, tw = routing[0].to(device).contiguous(), routing[1].to(device).contiguous()
    xq, xs = moe.quantize_nvfp4(x)
    n1, n2 = moe.transformed_weight_bytes_nvfp4(w.E, w.H, w.I)
    l1_t = torch.empty(n1, dtype=torch.uint8, device=device)
    l2_t = torch.empty(n2, dtype=torch.uint8, device=device)
    p1, p2 = n1 // w.E, n2 // w.E
    for e in range(w.E):
        a, b = moe.quantize_nvfp4(W.gen_l1(w, e, gen_device).to(device))
        c, d = moe.quantize_nvfp4(W.gen_l2(w, e, gen_device).to(device))
        moe.transform_weights_nvfp4(a[None], b[None], c[None], d[None],
                                    out=(l1_t[e * p1:(e + 1) * p1], l2_t[e * p2:(e + 1) * p2]))
    return dict(x=x, xq=xq, xs=xs, idx=idx, tw=tw, l1_t=l1_t, l2_t=l2_t)


def oracle_side_nvfp4(w: W.Workload, x_bf16: torch.Tensor, experts, gen_device="cuda"):
    """Oracle NVFP4 inputs from the same bf16 draws (listed experts only)."""
    xq, xs = oracle.quantize_nvfp4(x_bf16.float().cpu().numpy())
    experts = sorted(set(int(e) for e in experts))

    def quant(item):
        e, l1, l2 = item
        a, b = oracle.quantize_nvfp4(l1)
        c, d = oracle.quantize_nvfp4(l2)
        return e, (a, b, c, d)

    out = {}
    workers = max(1, min(len(experts), os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as pool:
        futs = [pool.submit(quant, (e, W.gen_l1(w, e, gen_device).float().cpu().numpy(),
                                    W.gen_l2(w, e, gen_device).float().cpu().numpy())) for e in experts]
        for f in futs:
            e, m = f.result()
            out[e] = m
    return xq, xs, out
