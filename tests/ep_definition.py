"""The expert-parallel dispatch and combine written out from their definition
(numpy, test-only): which routed slot goes to which rank and in which order,
and the top-k-weighted combine of the rows that come back.  Ranks own
contiguous expert ranges (rank r: experts [r E/R, (r+1) E/R)); the send order
is the routing's stable order, by expert and then by slot t*k+j."""
from __future__ import annotations

import numpy as np
import torch


def dispatch_plan(idx: np.ndarray, E: int, ranks: int):
    """idx i64 [T, k] -> (order, counts, eid, inv): ``order`` the slots t*k+j
    in send order (ids outside [0, E) dropped), ``counts`` i64 [ranks] rows per
    destination rank, ``eid`` the rows' local expert ids, ``inv`` i64 [T*k]
    each slot's row (-1: dropped)."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    slots = np.nonzero((flat >= 0) & (flat < E))[0]
    order = slots[np.argsort(flat[slots], kind="stable")]
    e_loc = E // ranks
    counts = np.bincount(flat[order] // e_loc, minlength=ranks).astype(np.int64)
    inv = np.full(flat.size, -1, np.int64)
    inv[order] = np.arange(order.size)
    return order, counts, flat[order] % e_loc, inv


def combine(rows: np.ndarray, inv: np.ndarray, topk_w: np.ndarray, k: int) -> torch.Tensor:
    """bf16 [T, H]: out[t] = bf16_rne(sum_{j ascending} w[t, j] * rows[inv[t*k+j]])
    with float32 products and sums; rows f32 [n, H] (bf16 values)."""
    w = np.asarray(topk_w, np.float32)
    T = w.shape[0]
    H = rows.shape[1] if rows.ndim == 2 else 0
    acc = np.zeros((T, H), np.float32)
    r = inv.reshape(T, k)
    for j in range(k):
        m = r[:, j] >= 0
        acc[m] += w[m, j:j + 1] * rows[r[m, j]]
    return torch.from_numpy(acc).to(torch.bfloat16)
