"""moe_forward_static, the entry point for callers that cannot allocate device
memory (inside CUDA graph capture, serving runtimes that own all device memory,
plug-ins without access to their host framework's allocator): its scratch is a
fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against moe_forward (the entry point with a caller
workspace) on the same inputs on two calls in a row (the array keeps the
previous call's contents): both run the same deterministic kernels, so the
outputs must be equal bit for bit, which also implies the layer's per-row
tolerance.  Also: the array's error word (moe_check_device_error_static)
reports a dropped out-of-range expert id and is cleared by the next call, and
a size beyond the array is rejected.  The conftest hook runs this file after
every other test.
"""
import numpy as np
import pytest
import torch

import workloads as W
from cases import MAX_ABS_TOL, REL_L2_TOL, gpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def within_tolerance(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    rn = np.linalg.norm(r, axis=1)
    nz = rn > 0
    assert np.all(g[~nz] == 0)
    rel = np.linalg.norm(g - r, axis=1)[nz] / rn[nz]
    mabs = np.abs(g - r).max(axis=1)[nz] / np.abs(r).max(axis=1)[nz]
    assert rel.max() <= REL_L2_TOL and mabs.max() <= MAX_ABS_TOL, (rel.max(), mabs.max())


CASES = [W.WORKLOADS[0], W.custom("static_mid", T=160, E=16, k=4, H=1024, I=512, seed=31)]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_static_matches_workspace_entry_point_two_calls_in_a_row(moe, w):
    g = gpu_layer(w)
    args = (g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I)
    ref = moe.forward(*args)
    first = moe.forward_static(*args)
    second = moe.forward_static(*args)
    torch.cuda.synchronize()
    assert moe.check_device_error_static() == 0
    assert torch.equal(first, ref)
    assert torch.equal(second, ref)
    within_tolerance(first, ref)


def test_static_error_word_reports_dropped_ids(moe):
    w = W.WORKLOADS[0]
    g = gpu_layer(w)
    bad = g["idx"].clone()
    bad[3, 1] = w.E + 5  # out of range: dropped from routing and reported
    args = (g["xq"], g["xs"], bad, g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I)
    ref = moe.forward(*args)
    got = moe.forward_static(*args)
    assert moe.check_device_error_static() == 5  # MOE_ERR_BAD_ROUTING
    assert torch.equal(got, ref)
    moe.forward_static(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I)
    assert moe.check_device_error_static() == 0
    assert moe.load().moe_check_device_error_static(-1, None) == 1  # MOE_ERR_INVALID_ARG


def test_static_rejects_sizes_beyond_its_array(moe):
    w = W.WORKLOADS[0]
    g = gpu_layer(w)
    T = 4096  # at H = 7168, I = 3072 this needs far more than the array holds
    H, I, E, k = 7168, 3072, 384, 6
    assert moe.workspace_bytes(T, E, k, H, I) > moe.STATIC_WORKSPACE_BYTES
    x = torch.zeros((T, H), dtype=torch.uint8, device="cuda")
    xs = torch.zeros((T, H // 32), dtype=torch.uint8, device="cuda")
    idx = torch.zeros((T, k), dtype=torch.int64, device="cuda")
    tw = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.forward_static(x, xs, idx, tw, g["l1_t"], g["l2_t"], E, H, I)
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
