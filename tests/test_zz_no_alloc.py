"""moe_forward_static, the entry point for callers that cannot allocate device
memory (inside CUDA graph capture, serving runtimes that own all device memory,
plug-ins without access to their host framework's allocator): its scratch is a
fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against moe_forward (the entry point with a caller
workspace) on the same inputs, within the layer's per-row tolerance, on two
calls in a row (the array keeps the previous call's contents), and the
rejection of a size beyond the array.  This file is collected last on purpose.
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
    within_tolerance(first, ref)
    within_tolerance(second, ref)


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
