"""Failure detection on the GPU without a fault: the library's bounded
device-side wait, run on a barrier that nothing completes with a 1 ms limit,
gives up, records the timeout in the workspace error word, and the context
stays usable (a forward on the same workspace afterwards is correct and
reports no error)."""
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


def test_bounded_wait_times_out_and_context_survives(moe):
    w = W.WORKLOADS[0]
    ws = torch.empty(moe.workspace_bytes(w.T, w.E, w.k, w.H, w.I), dtype=torch.uint8, device="cuda")
    moe.probe_wait_timeout(ws, timeout_us=1000)
    assert moe.check_device_error(ws) == 6                       # MOE_ERR_DEVICE_TIMEOUT
    hdr = ws[:16].view(torch.int32).cpu().numpy()
    assert hdr[0] & 2 and hdr[3] == 99                           # timeout bit, the probe's `where`
    # the context still works: a full forward on the same workspace is correct
    g = gpu_layer(w)
    out = moe.forward(g["xq"], g["xs"], g["idx"], g["tw"], g["l1_t"], g["l2_t"], w.E, w.H, w.I, workspace=ws)
    assert moe.check_device_error(ws) == 0
    idx = g["idx"].cpu().numpy()
    tok = np.arange(w.T)
    xq, xs, ex = oracle_side(w, g["x"], g["idx"], experts_of(idx, tok, w.E))
    ref = oracle.forward(xq, xs, idx, g["tw"].cpu().numpy(), ex, w.E, w.H, w.I)
    compare_rows(out, ref["out_bf16"], "after the probe")


def test_probe_rejects_bad_arguments(moe):
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    lib = moe.load()
    assert lib.moe_probe_wait_timeout(None, 4096, 1000, None) == 1
    assert lib.moe_probe_wait_timeout(ws.data_ptr(), 4096, 0, None) == 1
    assert lib.moe_probe_wait_timeout(ws.data_ptr(), 1024, 1000, None) == 3
