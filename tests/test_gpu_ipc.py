"""moe_ipc_handle on one GPU: the handle names the allocation that holds a
pointer and the offset locates the pointer inside it, so two views of one
allocation export the same handle with offsets that differ by the views'
distance.  (Opening a handle needs a second process on another GPU; the
exchange of handles and offsets between ranks is tested with gloo on CPU in
test_ep_peers_multiprocess.py.)"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_ipc_handle_names_the_allocation_and_the_offset(moelib):
    import moe_expert_layer_08_b200 as moe
    buf = torch.empty(8 << 20, dtype=torch.uint8, device="cuda")
    h0, o0 = moe.ipc_handle(buf)
    h1, o1 = moe.ipc_handle(buf[3 << 20:])
    assert len(h0) == moe.IPC_HANDLE_BYTES and h0 == h1
    assert o1 - o0 == 3 << 20
    other = torch.empty(8 << 20, dtype=torch.uint8, device="cuda")
    h2, _ = moe.ipc_handle(other)
    assert h2 != h0 or other.data_ptr() - buf.data_ptr() == _ - o0  # one caching-allocator block may hold both
    with pytest.raises(TypeError):
        moe.ipc_handle(torch.empty(4, dtype=torch.uint8))
