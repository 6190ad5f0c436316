"""CPU checks of the C ABI: the library loads, exports every function that
include/moe.h declares, and validates arguments on the host (before any CUDA
call, so these run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for need in ("moe_forward", "moe_transform_weights", "moe_workspace_bytes", "moe_read_routing",
                 "moe_check_device_error", "moe_quantize_fp8", "moe_quantize_fp4"):
        assert need in names


def test_library_exports_every_declared_symbol(moelib):
    for name in declared_functions():
        assert hasattr(moelib, name), name


def test_status_strings(moelib):
    assert moelib.moe_status_string(0) == b"MOE_OK"
    assert moelib.moe_status_string(3) == b"MOE_ERR_WORKSPACE_TOO_SMALL"
    assert moelib.moe_status_string(99) == b"MOE_ERR_UNKNOWN"
    assert moelib.moe_abi_version() >= 1


def test_sizes_are_host_only_and_consistent(moelib):
    import moe_expert_layer_08_b200 as m
    l1, l2 = m.transformed_weight_bytes(384, 7168, 3072)
    per_expert = (2 * 3072 * 7168 + 7168 * 3072) // 2 + (2 * 3072 * 7168 + 7168 * 3072) // 32
    assert l1 + l2 == 384 * per_expert == 384 * 35094528
    a = m.workspace_bytes(8, 384, 6, 7168, 3072)
    b = m.workspace_bytes(8192, 384, 6, 7168, 3072)
    assert 0 < a < b
    assert m.workspace_bytes(0, 8, 2, 256, 256) > 0


def test_forward_kernel_launches(moelib):
    """One-block routing up to T*k = 1024 routed rows (2 kernels), block-scan
    routing above (5), plus GEMM1, GEMM2 and the combine; above T*k = 8E
    (160-row chunks) GEMM1 and GEMM2 run once more over the side list of
    lightly loaded experts; nothing for T = 0."""
    import moe_expert_layer_08_b200 as m
    assert m.forward_kernel_launches(8, 384, 6, 7168, 3072) == 5
    assert m.forward_kernel_launches(170, 384, 6, 7168, 3072) == 5     # 1020 rows
    assert m.forward_kernel_launches(171, 384, 6, 7168, 3072) == 8     # 1026 rows
    assert m.forward_kernel_launches(512, 384, 6, 7168, 3072) == 8     # 3072 rows = 8E: 32-row chunks
    assert m.forward_kernel_launches(513, 384, 6, 7168, 3072) == 10    # side list
    assert m.forward_kernel_launches(8192, 384, 6, 7168, 3072) == 10
    assert m.forward_kernel_launches(64, 8, 2, 256, 256) == 7          # one-block routing, side list
    assert m.forward_kernel_launches(0, 8, 2, 256, 256) == 0
    with pytest.raises(m.MoEError):
        m.forward_kernel_launches(4, 8, 9, 256, 256)                   # k > E
    with pytest.raises(m.MoEError):
        m.forward_kernel_launches(4, 8, 2, 200, 256)                   # H % 128


@pytest.mark.parametrize("E,H,I,status", [(8, 200, 256, 2), (8, 256, 200, 2), (8, 256, 8320, 2),
                                          (2000, 256, 256, 2), (0, 256, 256, 1)])
def test_bad_shapes_fail_closed(moelib, E, H, I, status):
    import moe_expert_layer_08_b200 as m
    with pytest.raises(m.MoEError) as ei:
        m.transformed_weight_bytes(E, H, I)
    assert ei.value.status == status
    n = ctypes.c_size_t()
    assert moelib.moe_workspace_bytes(4, E, 2, H, I, ctypes.byref(n)) == status


def test_forward_validation_before_any_cuda_call(moelib):
    f = moelib.moe_forward
    p = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    # unsupported shape
    assert f(p, p, p, p, p, p, p, 4, 8, 2, 200, 256, p, 1 << 30, None, None, None) == 2
    # k > E, negative T
    assert f(p, p, p, p, p, p, p, 4, 8, 9, 256, 256, p, 1 << 30, None, None, None) == 1
    assert f(p, p, p, p, p, p, p, -1, 8, 2, 256, 256, p, 1 << 30, None, None, None) == 1
    # T = 0 is a no-op
    assert f(None, None, None, None, None, None, None, 0, 8, 2, 256, 256, None, 0, None, None, None) == 0
    # null / misaligned pointers
    assert f(None, p, p, p, p, p, p, 4, 8, 2, 256, 256, p, 1 << 30, None, None, None) == 1
    q = ctypes.c_void_p(0x10001)
    assert f(q, p, p, p, p, p, p, 4, 8, 2, 256, 256, p, 1 << 30, None, None, None) == 1
    # workspace too small
    assert f(p, p, p, p, p, p, p, 4, 8, 2, 256, 256, p, 16, None, None, None) == 3


def test_quantize_and_transform_validation(moelib):
    p = ctypes.c_void_p(0x10000)
    assert moelib.moe_quantize_fp8(p, 4, 33, p, p, None) == 2
    assert moelib.moe_quantize_fp4(p, -1, 32, p, p, None) == 1
    assert moelib.moe_quantize_fp8(None, 0, 32, None, None, None) == 0
    assert moelib.moe_transform_weights(p, p, p, p, 4, 256, 200, p, p, None) == 2
    assert moelib.moe_transform_weights(None, p, p, p, 4, 256, 256, p, p, None) == 1
    odd = ctypes.c_void_p(0x10080)  # 128- but not 256-byte aligned destination
    assert moelib.moe_transform_weights(p, p, p, p, 4, 256, 256, odd, p, None) == 1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import moe_expert_layer_08_b200 as m
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(m, "_lib", None)
    with pytest.raises(ImportError):
        m.load()


def test_static_entry_point_rejects_oversize_before_any_cuda_call(moelib):
    p = ctypes.c_void_p(0x10000)
    # T = 4096 at E = 384, top-6, H = 7168, I = 3072 does not fit the fixed array
    assert moelib.moe_forward_static(p, p, p, p, p, p, p, 4096, 384, 6, 7168, 3072, None, None, None) == 3
    assert moelib.moe_forward_static(p, p, p, p, p, p, p, 4, 8, 2, 200, 256, None, None, None) == 2
    assert moelib.moe_forward_static(None, None, None, None, None, None, None, 0, 8, 2, 256, 256,
                                     None, None, None) == 0


def test_forward_act_validates_activation_before_any_cuda_call(moelib):
    import moe_expert_layer_08_b200 as m
    p = ctypes.c_void_p(0x10000)
    f = moelib.moe_forward_act
    for kind, beta, lb in ((1, 0.0, 1.0), (1, -2.0, 0.0), (1, float("inf"), 0.0), (1, 1.0, -1.0),
                           (1, 1.0, float("nan")), (7, 1.0, 0.0)):
        a = m.Activation(kind, beta, lb)
        assert f(p, p, p, p, p, p, p, 4, 8, 2, 256, 256, p, 16, None, None, ctypes.byref(a), None) == 1
    # a valid activation passes to the next check (workspace too small)
    a = m.activation("situ", 1.25, 1.5)
    assert f(p, p, p, p, p, p, p, 4, 8, 2, 256, 256, p, 16, None, None, ctypes.byref(a), None) == 3


def test_layouts_and_scale_transform_validate_on_the_host(moelib):
    """Row-major layout entry points: sizes, and every bad argument rejected
    before any CUDA call."""
    import moe_expert_layer_08_b200 as m
    l1, l2 = m.transformed_weight_bytes(384, 7168, 3072)
    s1, s2 = m.transformed_scale_bytes(384, 7168, 3072)
    assert (s1 * 17, s2 * 17) == (l1, l2)           # one 512-byte block per 8704-byte packet
    assert m.transformed_scale_bytes(2, 384, 128) == (2 * 1 * 3 * 2 * 512, 2 * 2 * 1 * 2 * 512)  # odd H tiles pad
    n = ctypes.c_size_t()
    assert moelib.moe_transformed_scale_bytes(8, 200, 256, ctypes.byref(n), ctypes.byref(n)) == 2
    p = ctypes.c_void_p(256)
    assert moelib.moe_transform_scales(None, p, 8, 256, 256, p, p, None) == 1
    assert moelib.moe_transform_scales(p, p, 8, 256, 256, ctypes.c_void_p(260), p, None) == 1   # misaligned out
    args = lambda wts: (p, p, p, p, wts, p, 4, 8, 2, 256, 256, p, 1 << 30, None, None, None, None)
    assert moelib.moe_forward_weights(*args(None)) == 1
    assert moelib.moe_forward_weights(*args(ctypes.byref(m.Weights(7, 256, 0, 256, 0)))) == 1   # unknown layout
    assert moelib.moe_forward_weights(*args(ctypes.byref(m.Weights(0, 256, 256, 256, 0)))) == 1  # packets + scales
    assert moelib.moe_forward_weights(*args(ctypes.byref(m.Weights(1, 256, 0, 256, 256)))) == 1  # row-major, no l1_sf
    assert moelib.moe_forward_weights(*args(ctypes.byref(m.Weights(1, 256, 300, 256, 256)))) == 1  # misaligned
    assert moelib.moe_forward_weights(*args(ctypes.byref(m.Weights(1, 0, 256, 256, 256)))) == 1  # no body


def test_nvfp4_entry_points_validate_on_the_host(moelib):
    import moe_expert_layer_08_b200 as m
    a, b = m.transformed_weight_bytes_nvfp4(384, 7168, 3072)
    assert (a, b) == (384 * 24 * 28 * 2 * 18432, 384 * 28 * 12 * 2 * 18432)
    n = ctypes.c_size_t()
    assert moelib.moe_transformed_weight_bytes_nvfp4(8, 384, 256, ctypes.byref(n), ctypes.byref(n)) == 2  # H % 256
    assert moelib.moe_transformed_weight_bytes_nvfp4(8, 256, 384, ctypes.byref(n), ctypes.byref(n)) == 2  # I % 256
    p = ctypes.c_void_p(256)
    assert moelib.moe_quantize_nvfp4(p, 4, 40, p, p, None) == 2               # cols % 16
    assert moelib.moe_quantize_nvfp4(None, 4, 32, p, p, None) == 1
    assert moelib.moe_transform_weights_nvfp4(p, p, p, None, 2, 256, 256, p, p, None) == 1
    args = lambda **kw: [kw.get("x", p), p, p, p, p, p, p, kw.get("T", 4), 8, kw.get("k", 2), kw.get("H", 256), 256,
                         p, 1 << 30, None, None, None, None]
    assert moelib.moe_forward_nvfp4(*args(H=384)) == 2
    assert moelib.moe_forward_nvfp4(*args(k=9)) == 1
    assert moelib.moe_forward_nvfp4(*args(x=ctypes.c_void_p(264))) == 1      # misaligned x
    assert moelib.moe_forward_nvfp4(*args(T=0)) == 0


def test_shared_expert_entry_points_validate_on_the_host(moelib):
    """Workspace size = 2 KiB header + h [T, SI] bf16 (256-aligned) + the
    K-split partial sums (up to 64 tokens: 256 units of 32-token blocks, 8
    MiB; up to 128: 256 units of 64-token blocks, 16 MiB; above: 160 units of
    128-token blocks, 20 MiB); shapes, token counts, activations and sizes are
    checked before any CUDA call."""
    import ctypes
    import moe_expert_layer_08_b200 as m
    lib = m.load()
    scratch32 = 256 * 2 * 32 * 128 * 4
    scratch64 = 256 * 2 * 64 * 128 * 4
    scratch128 = 160 * 2 * 128 * 128 * 4
    assert m.shared_workspace_bytes(8192, 7168, 2048) == 2048 + 8192 * 2048 * 2 + scratch128
    assert m.shared_workspace_bytes(129, 7168, 2048) == 2048 + 129 * 2048 * 2 + scratch128
    assert m.shared_workspace_bytes(128, 7168, 2048) == 2048 + 128 * 2048 * 2 + scratch64
    assert m.shared_workspace_bytes(65, 7168, 2048) == 2048 + 65 * 2048 * 2 + scratch64
    assert m.shared_workspace_bytes(64, 7168, 2048) == 2048 + 64 * 2048 * 2 + scratch32
    assert m.shared_workspace_bytes(3, 256, 128) == 2048 + 768 + scratch32
    assert m.shared_workspace_bytes(0, 256, 128) == 2048 + scratch32
    n = ctypes.c_size_t()
    assert lib.moe_shared_workspace_bytes(8, 200, 128, ctypes.byref(n)) == 2   # SH % 128
    assert lib.moe_shared_workspace_bytes(8, 256, 100, ctypes.byref(n)) == 2   # SI % 128
    assert lib.moe_shared_workspace_bytes(-1, 256, 128, ctypes.byref(n)) == 1
    f = lib.moe_shared_forward
    assert f(None, None, None, None, 0, 256, 128, None, None, 0, None) == 0     # T = 0: nothing to do
    assert f(None, None, None, None, 4, 256, 128, None, None, 0, None) == 1     # null pointers
    assert f(None, None, None, None, 4, 200, 128, None, None, 0, None) == 2     # SH % 128
    assert f(None, None, None, None, -1, 256, 128, None, None, 0, None) == 1
    bad = m.Activation(1, 0.0, 0.0)                                             # SiTU needs beta > 0
    assert f(None, None, None, None, 4, 256, 128, ctypes.byref(bad), None, 0, None) == 1
    fake = ctypes.c_void_p(1 << 20)                                            # never dereferenced
    assert f(fake, fake, fake, fake, 4, 256, 128, None, fake, 16, None) == 3   # workspace too small


def test_workspace_grows_monotonically_with_T(moelib):
    """A workspace sized for T_max serves every T <= T_max, across the switch
    from 32-row to 160-row chunks (T*k > 8E) and the side list's regions."""
    import moe_expert_layer_08_b200 as m
    for E, k, H, I in ((8, 2, 256, 256), (64, 6, 1024, 512), (384, 6, 7168, 3072)):
        sizes = [m.workspace_bytes(T, E, k, H, I) for T in range(0, 1200, 7)]
        assert all(a <= b for a, b in zip(sizes, sizes[1:])), (E, k, H, I)


def test_static_workspace_holds_decode_batches(moelib):
    """The fixed scratch of moe_forward_static holds T = 128 tokens at E = 384,
    top-6, H = 7168, I = 3072 (the sizes its documentation names)."""
    import moe_expert_layer_08_b200 as m
    assert m.workspace_bytes(128, 384, 6, 7168, 3072) <= m.STATIC_WORKSPACE_BYTES


def test_expert_parallel_entry_points_validate_on_the_host(moelib):
    """The dispatch workspace holds the routing metadata only (monotone in T,
    a small fraction of the layer's); shapes, rank counts, pointers,
    alignment and sizes are checked before any CUDA call."""
    import moe_expert_layer_08_b200 as m
    lib = m.load()
    sizes = [m.ep_workspace_bytes(T, 384, 6, 7168) for T in range(0, 9000, 97)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    assert m.ep_workspace_bytes(8192, 384, 6, 7168) < m.workspace_bytes(8192, 384, 6, 7168, 3072) // 100
    n = ctypes.c_size_t()
    assert lib.moe_ep_workspace_bytes(8, 384, 6, 200, ctypes.byref(n)) == 2    # H % 128
    assert lib.moe_ep_workspace_bytes(8, 4, 6, 256, ctypes.byref(n)) == 1      # k > E
    assert lib.moe_ep_workspace_bytes(8, 4, 2, 256, None) == 1
    p = ctypes.c_void_p(1 << 20)                                               # never dereferenced

    def dispatch(**kw):
        return lib.moe_ep_dispatch(kw.get("x", p), p, p, kw.get("T", 4), 8, 2, kw.get("H", 256),
                                   kw.get("ranks", 2), kw.get("ws", p), kw.get("ws_bytes", 1 << 30), p, p, p,
                                   kw.get("counts", p), None)

    assert dispatch(ranks=0) == 1
    assert dispatch(ranks=9) == 1                                  # more ranks than experts
    assert dispatch(ranks=3) == 2                                  # E % ranks
    assert dispatch(H=200) == 2
    assert dispatch(T=-1) == 1
    assert dispatch(ws=None) == 1
    assert dispatch(counts=None) == 1
    assert dispatch(x=ctypes.c_void_p((1 << 20) + 8)) == 1         # x not 16-byte aligned
    assert dispatch(ws_bytes=16) == 3

    def combine(**kw):
        return lib.moe_ep_combine(kw.get("y", p), p, kw.get("T", 4), 8, 2, 256, kw.get("ws", p),
                                  kw.get("ws_bytes", 1 << 30), p, None)

    assert combine(T=0) == 0                                       # nothing to do
    assert combine(T=-1) == 1
    assert combine(y=None) == 1
    assert combine(ws_bytes=16) == 3

    def peers(**kw):
        return lib.moe_ep_combine_peers(kw.get("peer_y", p), kw.get("base", p), p, p, kw.get("T", 4), 8, 2, 256,
                                        kw.get("ranks", 2), p, kw.get("ws_bytes", 1 << 30), kw.get("out", p), None)

    assert peers(T=0) == 0
    assert peers(ranks=3) == 2
    assert peers(ranks=0) == 1
    assert peers(peer_y=None) == 1
    assert peers(base=ctypes.c_void_p((1 << 20) + 4)) == 1                  # recv_base not 8-byte aligned
    assert peers(out=ctypes.c_void_p((1 << 20) + 8)) == 1                   # out not 16-byte aligned
    assert peers(ws_bytes=16) == 3

    def route(**kw):
        return lib.moe_ep_route(kw.get("idx", p), kw.get("T", 4), 8, 2, 256, kw.get("ranks", 2), kw.get("ws", p),
                                kw.get("ws_bytes", 1 << 30), kw.get("counts", p), None)

    assert route(ranks=3) == 2
    assert route(idx=None) == 1
    assert route(counts=None) == 1
    assert route(ws_bytes=16) == 3

    def push(**kw):
        return lib.moe_ep_dispatch_peers(p, p, p, kw.get("T", 4), 8, 2, 256, kw.get("ranks", 2), p,
                                         kw.get("ws_bytes", 1 << 30), kw.get("px", p), p, p, p, None)

    assert push(T=0) == 0
    assert push(ranks=3) == 2
    assert push(px=None) == 1
    assert push(px=ctypes.c_void_p((1 << 20) + 4)) == 1                     # pointer table not 8-byte aligned
    assert push(ws_bytes=16) == 3
