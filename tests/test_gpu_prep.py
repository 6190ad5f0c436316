"""GPU checks of the preparation kernels and the routing through the C ABI:
quantisers bit-exact against the oracle's, the weight-packet transform against
a host-side un-transform, routing metadata bit-exact against the oracle's
stable counting sort."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(moelib):
    import moe_expert_layer_08_b200 as m
    return m


def special_rows(cols, gen):
    rows = [torch.zeros(cols)]
    r = torch.randn(cols, generator=gen) * 1e-3
    r[0] = 1.0
    r[1:32] = -1e-30                         # negatives that round to -0
    rows.append(r)
    rows.append(torch.randn(cols, generator=gen) * 3e4)
    r = torch.randn(cols, generator=gen)
    r[5] = 448.0                             # exactly on a scale boundary
    r[min(40, cols - 1)] = 6.0
    rows.append(r)
    rows.append(torch.full((cols,), -0.0))
    return torch.stack(rows)


@pytest.mark.parametrize("rows,cols", [(1, 32), (257, 512), (64, 7168)])
def test_quantize_fp8_matches_oracle(moe, rows, cols):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    x = torch.cat([torch.randn((rows, cols), generator=g) * 0.5, special_rows(cols, g)]).to(torch.bfloat16)
    q, sf = moe.quantize_fp8(x.cuda())
    rq, rsf = oracle.quantize_e4m3(x.float().numpy())
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(q.cpu().numpy(), rq)


@pytest.mark.parametrize("rows,cols", [(3, 64), (300, 256), (128, 3072)])
def test_quantize_fp4_matches_oracle(moe, rows, cols):
    g = torch.Generator().manual_seed(rows * 11 + cols)
    x = torch.cat([torch.randn((rows, cols), generator=g) * 0.04, special_rows(cols, g)]).to(torch.bfloat16)
    q, sf = moe.quantize_fp4(x.cuda())
    rq, rsf = oracle.quantize_e2m1(x.float().numpy())
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(q.cpu().numpy(), rq)


def untransform(l1_t, l2_t, E, H, I):
    """Host inverse of the packet layout: packets of a 128x128 tile (64-byte
    rows) followed by 512 scale bytes (lane r%32, word r//32 holds row r's 4
    scale bytes).  L1: expert -> I-tile -> K tile -> (gate, up); L2: expert ->
    H-tile pair -> K tile -> (tile 2p, tile 2p+1), padded to an even count."""
    P = 8704

    def unpack(buf, rows_per_expert, K, groups, row_of):
        KB = K // 128
        pk = buf.reshape(E, groups, KB, 2, P)
        w = np.zeros((E, rows_per_expert, K // 2), np.uint8)
        s = np.zeros((E, rows_per_expert, K // 32), np.uint8)
        body = pk[..., :8192].reshape(E, groups, KB, 2, 128, 64)
        sfb = pk[..., 8192:].reshape(E, groups, KB, 2, 32, 4, 4)  # lane, word, byte
        for g in range(groups):
            for slot in range(2):
                r0 = row_of(g, slot)
                if r0 >= rows_per_expert:
                    assert not body[:, g, :, slot].any() and not sfb[:, g, :, slot].any()  # zero padding
                    continue
                rows = slice(r0, r0 + 128)
                w[:, rows, :] = body[:, g, :, slot].transpose(0, 2, 1, 3).reshape(E, 128, K // 2)
                for kb in range(KB):
                    v = sfb[:, g, kb, slot]  # [E, lane, word, byte]
                    s[:, rows, kb * 4:kb * 4 + 4] = v.transpose(0, 2, 1, 3).reshape(E, 128, 4)
        return w, s

    w1, s1 = unpack(l1_t, 2 * I, H, I // 128, lambda g, slot: slot * I + g * 128)
    w2, s2 = unpack(l2_t, H, I, (H // 128 + 1) // 2, lambda g, slot: (2 * g + slot) * 128)
    return w1, s1, w2, s2


@pytest.mark.parametrize("E,H,I", [(1, 128, 128), (3, 256, 384), (2, 512, 256), (2, 384, 128)])
def test_transform_round_trip(moe, E, H, I):
    g = torch.Generator().manual_seed(E + H + I)
    l1 = torch.randint(0, 256, (E, 2 * I, H // 2), generator=g, dtype=torch.uint8)
    l1s = torch.randint(0, 256, (E, 2 * I, H // 32), generator=g, dtype=torch.uint8)
    l2 = torch.randint(0, 256, (E, H, I // 2), generator=g, dtype=torch.uint8)
    l2s = torch.randint(0, 256, (E, H, I // 32), generator=g, dtype=torch.uint8)
    a, b = moe.transform_weights(l1.cuda(), l1s.cuda(), l2.cuda(), l2s.cuda())
    n1, n2 = moe.transformed_weight_bytes(E, H, I)
    assert a.numel() == n1 and b.numel() == n2
    w1, s1, w2, s2 = untransform(a.cpu().numpy(), b.cpu().numpy(), E, H, I)
    assert np.array_equal(w1, l1.numpy()) and np.array_equal(s1, l1s.numpy())
    assert np.array_equal(w2, l2.numpy()) and np.array_equal(s2, l2s.numpy())


def route_through_forward(moe, T, k, E, idx, H=128, I=128):
    """Run a (tiny-weight) forward to populate the workspace, return its routing."""
    w = W.custom("r", T=T, E=E, k=k, H=H, I=I, seed=5)
    x = torch.randn((T, H), device="cuda").to(torch.bfloat16)
    xq, xs = moe.quantize_fp8(x)
    n1, n2 = moe.transformed_weight_bytes(E, H, I)
    l1_t = torch.zeros(n1, dtype=torch.uint8, device="cuda")
    l2_t = torch.zeros(n2, dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.workspace_bytes(T, E, k, H, I), dtype=torch.uint8, device="cuda")
    tw = torch.ones((T, k), dtype=torch.float32, device="cuda")
    out = moe.forward(xq, xs, idx.cuda(), tw, l1_t, l2_t, E, H, I, workspace=ws)
    status = moe.check_device_error(ws)
    return moe.read_routing(ws, T, E, k, H, I), status, out


ROUTING_CASES = [
    ("uniform", 64, 2, 8), ("uniform", 8, 6, 384), ("uniform", 1000, 6, 384), ("uniform", 8192, 6, 384),
    ("zipf", 4096, 8, 256), ("structured", 96, 4, 12), ("one_expert", 300, 1, 5), ("dups", 77, 3, 3),
]


@pytest.mark.parametrize("kind,T,k,E", ROUTING_CASES)
def test_routing_bit_exact(moe, kind, T, k, E):
    if kind in ("uniform", "zipf"):
        idx, _ = W.gen_routing(W.custom(kind, T=T, E=E, k=k, H=128, I=128, seed=T, routing=kind))
    elif kind == "structured":
        idx, _ = W.structured_routing(T, k, E)
    elif kind == "one_expert":
        idx = torch.full((T, k), 3, dtype=torch.int64)
    else:
        idx = torch.randint(0, E, (T, k), generator=torch.Generator().manual_seed(1), dtype=torch.int64)
    got, status, _ = route_through_forward(moe, T, k, E, idx)
    ref = oracle.route(idx.numpy(), E)
    assert status == 0
    for key in ("count", "offset", "perm", "inv"):
        assert np.array_equal(got[key].numpy(), ref[key]), key


def test_out_of_range_ids_are_dropped_and_reported(moe):
    T, k, E = 50, 3, 7
    idx = torch.randint(0, E, (T, k), generator=torch.Generator().manual_seed(2), dtype=torch.int64)
    idx[3, 1] = E
    idx[10, 0] = -1
    idx[49, 2] = 1 << 40
    got, status, _ = route_through_forward(moe, T, k, E, idx)
    ref = oracle.route(idx.numpy(), E)
    assert ref["dropped"] == 3
    assert status == moe_status("MOE_ERR_BAD_ROUTING")
    for key in ("count", "offset", "perm", "inv"):
        assert np.array_equal(got[key].numpy(), ref[key]), key


def moe_status(name):
    import moe_expert_layer_08_b200 as m
    return {v: k for k, v in m.STATUS.items()}[name]
