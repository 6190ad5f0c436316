"""B200 (sm_100a) FP8 x FP4 MoE expert layer -- Python binding of include/moe.h.

Every entry point of the C ABI has a function of the same name here (without
the ``moe_`` prefix).  This module only marshals torch tensors into pointers
and sizes and allocates outputs with torch; every step of the layer runs in the
CUDA library ``libmoe_b200.so`` next to this file.  There is no fallback: if
the library is missing, loading fails with an error naming the build command.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "MoEError", "load", "status_string", "abi_version", "quantize_fp8", "quantize_fp4",
    "transformed_weight_bytes", "transform_weights", "workspace_bytes", "forward",
    "read_routing", "check_device_error", "MoELayer", "NUM_STAGE_EVENTS", "STATUS",
    "forward_static", "check_device_error_static", "STATIC_WORKSPACE_BYTES", "Activation", "activation", "forward_kernel_launches",
    "Weights", "RowMajorWeights", "transformed_scale_bytes", "transform_scales", "LAYOUT_PACKETS",
    "LAYOUT_ROW_MAJOR", "quantize_nvfp4", "transformed_weight_bytes_nvfp4", "transform_weights_nvfp4",
    "forward_nvfp4", "shared_workspace_bytes", "shared_workspace", "shared_forward", "probe_wait_timeout",
    "ep_workspace_bytes", "ep_dispatch", "ep_combine", "ep_combine_peers", "ep_route", "ep_dispatch_peers",
    "ipc_handle", "ipc_open", "ipc_close", "IPC_HANDLE_BYTES",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
IPC_HANDLE_BYTES = 64  # MOE_IPC_HANDLE_BYTES
NUM_STAGE_EVENTS = 5
STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024  # MOE_STATIC_WORKSPACE_BYTES
STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_BAD_ROUTING",
    6: "MOE_ERR_DEVICE_TIMEOUT",
}

_lib = None
_lock = threading.Lock()


class Activation(ctypes.Structure):
    """moe_activation_t: kind 0 = SwiGLU, 1 = SiTU (beta, linear_beta; 0 = absent)."""
    _fields_ = [("kind", ctypes.c_int), ("beta", ctypes.c_float), ("linear_beta", ctypes.c_float)]


LAYOUT_PACKETS, LAYOUT_ROW_MAJOR = 0, 1


class Weights(ctypes.Structure):
    """moe_weights_t: a weight layout and its four pointers."""
    _fields_ = [("layout", ctypes.c_int), ("l1", ctypes.c_void_p), ("l1_sf", ctypes.c_void_p),
                ("l2", ctypes.c_void_p), ("l2_sf", ctypes.c_void_p)]


class RowMajorWeights:
    """Weights in the row-major layout: the FP4 bodies as quantize_fp4 wrote them
    (l1 [E, 2I, H/2], l2 [E, H, I/2], u8) and the scale blocks of
    transform_scales (1-D u8).  Holds the tensors so they outlive the calls."""

    def __init__(self, l1, l1_sf_t, l2, l2_sf_t):
        for t, n in ((l1, "l1"), (l2, "l2")):
            _need(t, torch.uint8, n, 3)
        _need(l1_sf_t, torch.uint8, "l1_sf_t")
        _need(l2_sf_t, torch.uint8, "l2_sf_t")
        self.l1, self.l1_sf_t, self.l2, self.l2_sf_t = l1, l1_sf_t, l2, l2_sf_t

    def struct(self) -> Weights:
        return Weights(LAYOUT_ROW_MAJOR, _ptr(self.l1), _ptr(self.l1_sf_t), _ptr(self.l2), _ptr(self.l2_sf_t))


def activation(kind: str = "swiglu", beta: float = 1.0, linear_beta=None) -> Activation:
    return Activation({"swiglu": 0, "situ": 1}[kind], float(beta), float(linear_beta or 0.0))


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def _declare(lib):
    c = ctypes
    P, I32, I64, SZ = c.c_void_p, c.c_int, c.c_int64, c.c_size_t
    sig = {
        "moe_status_string": (c.c_char_p, [I32]),
        "moe_abi_version": (I32, []),
        "moe_quantize_fp8": (I32, [P, I64, I64, P, P, P]),
        "moe_quantize_fp4": (I32, [P, I64, I64, P, P, P]),
        "moe_transformed_weight_bytes": (I32, [I32, I32, I32, c.POINTER(SZ), c.POINTER(SZ)]),
        "moe_transform_weights": (I32, [P, P, P, P, I32, I32, I32, P, P, P]),
        "moe_workspace_bytes": (I32, [I32, I32, I32, I32, I32, c.POINTER(SZ)]),
        "moe_forward_kernel_launches": (I32, [I32, I32, I32, I32, I32, c.POINTER(I32)]),
        "moe_forward": (I32, [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P, P]),
        "moe_read_routing": (I32, [P, I32, I32, I32, I32, I32, P, P, P, P, P]),
        "moe_check_device_error": (I32, [P, P]),
        "moe_forward_static": (I32, [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, P, P, P]),
        "moe_check_device_error_static": (I32, [I32, P]),
        "moe_forward_act": (I32, [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P,
                                  c.POINTER(Activation), P]),
        "moe_transformed_scale_bytes": (I32, [I32, I32, I32, c.POINTER(SZ), c.POINTER(SZ)]),
        "moe_quantize_nvfp4": (I32, [P, I64, I64, P, P, P]),
        "moe_transformed_weight_bytes_nvfp4": (I32, [I32, I32, I32, c.POINTER(SZ), c.POINTER(SZ)]),
        "moe_transform_weights_nvfp4": (I32, [P, P, P, P, I32, I32, I32, P, P, P]),
        "moe_forward_nvfp4": (I32, [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P,
                                    c.POINTER(Activation), P]),
        "moe_transform_scales": (I32, [P, P, I32, I32, I32, P, P, P]),
        "moe_forward_weights": (I32, [P, P, P, P, c.POINTER(Weights), P, I32, I32, I32, I32, I32, P, SZ, P, P,
                                      c.POINTER(Activation), P]),
        "moe_shared_workspace_bytes": (I32, [I32, I32, I32, c.POINTER(SZ)]),
        "moe_probe_wait_timeout": (I32, [P, SZ, c.c_uint, P]),
        "moe_shared_forward": (I32, [P, P, P, P, I32, I32, I32, c.POINTER(Activation), P, SZ, P]),
        "moe_ep_workspace_bytes": (I32, [I32, I32, I32, I32, c.POINTER(SZ)]),
        "moe_ep_dispatch": (I32, [P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P, P, P, P]),
        "moe_ep_combine": (I32, [P, P, I32, I32, I32, I32, P, SZ, P, P]),
        "moe_ep_combine_peers": (I32, [P, P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P]),
        "moe_ep_route": (I32, [P, I32, I32, I32, I32, I32, P, SZ, P, P]),
        "moe_ep_dispatch_peers": (I32, [P, P, P, I32, I32, I32, I32, I32, P, SZ, P, P, P, P, P]),
        "moe_ipc_handle": (I32, [P, P, c.POINTER(SZ)]),
        "moe_ipc_open": (I32, [P, I32, c.POINTER(P)]),
        "moe_ipc_close": (I32, [P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def load():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing; build it with `python -m moe_expert_layer_08_b200.build`")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise MoEError(status, what)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def abi_version() -> int:
    return load().moe_abi_version()


def quantize_fp8(x: torch.Tensor, stream=None):
    """bf16 [rows, cols] -> (E4M3 codes u8 [rows, cols], UE8M0 u8 [rows, cols/32])."""
    _need(x, torch.bfloat16, "x", 2)
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    sf = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device)
    _check(load().moe_quantize_fp8(_ptr(x), rows, cols, _ptr(q), _ptr(sf), _stream(stream)), "moe_quantize_fp8")
    return q, sf


def quantize_fp4(w: torch.Tensor, stream=None):
    """bf16 [rows, cols] -> (packed E2M1 u8 [rows, cols/2], UE8M0 u8 [rows, cols/32])."""
    _need(w, torch.bfloat16, "w", 2)
    rows, cols = w.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    sf = torch.empty((rows, cols // 32), dtype=torch.uint8, device=w.device)
    _check(load().moe_quantize_fp4(_ptr(w), rows, cols, _ptr(q), _ptr(sf), _stream(stream)), "moe_quantize_fp4")
    return q, sf


def transformed_weight_bytes(E: int, H: int, I: int):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().moe_transformed_weight_bytes(E, H, I, ctypes.byref(a), ctypes.byref(b)),
           "moe_transformed_weight_bytes")
    return a.value, b.value


def transform_weights(l1, l1_sf, l2, l2_sf, out=None, stream=None):
    """[E, 2I, H/2], [E, 2I, H/32], [E, H, I/2], [E, H, I/32] (u8) -> (l1_t, l2_t)
    tile-packet buffers (u8, 1-D).  ``out`` may give the two destination views."""
    for t, n in ((l1, "l1"), (l1_sf, "l1_sf"), (l2, "l2"), (l2_sf, "l2_sf")):
        _need(t, torch.uint8, n, 3)
    E, twoI, Hh = l1.shape
    H, I = Hh * 2, twoI // 2
    if l1_sf.shape != (E, 2 * I, H // 32) or l2.shape != (E, H, I // 2) or l2_sf.shape != (E, H, I // 32):
        raise ValueError("inconsistent weight shapes")
    n1, n2 = transformed_weight_bytes(E, H, I)
    if out is None:
        l1_t = torch.empty(n1, dtype=torch.uint8, device=l1.device)
        l2_t = torch.empty(n2, dtype=torch.uint8, device=l1.device)
    else:
        l1_t, l2_t = out
        if l1_t.numel() < n1 or l2_t.numel() < n2:
            raise ValueError("output buffers too small")
    _check(load().moe_transform_weights(_ptr(l1), _ptr(l1_sf), _ptr(l2), _ptr(l2_sf), E, H, I,
                                        _ptr(l1_t), _ptr(l2_t), _stream(stream)), "moe_transform_weights")
    return l1_t, l2_t


def quantize_nvfp4(x, stream=None):
    """bf16 [rows, cols] -> (packed E2M1 u8 [rows, cols/2], UE4M3 scales u8 [rows, cols/16])."""
    _need(x, torch.bfloat16, "x", 2)
    rows, cols = x.shape
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    _check(load().moe_quantize_nvfp4(_ptr(x), rows, cols, _ptr(q), _ptr(sf), _stream(stream)), "moe_quantize_nvfp4")
    return q, sf


def transformed_weight_bytes_nvfp4(E: int, H: int, I: int):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().moe_transformed_weight_bytes_nvfp4(E, H, I, ctypes.byref(a), ctypes.byref(b)),
           "moe_transformed_weight_bytes_nvfp4")
    return a.value, b.value


def transform_weights_nvfp4(l1, l1_sf, l2, l2_sf, out=None, stream=None):
    """[E, 2I, H/2], [E, 2I, H/16], [E, H, I/2], [E, H, I/16] (u8) -> (l1_t, l2_t)
    NVFP4 packet buffers (u8, 1-D).  ``out`` may give the two destination views."""
    for t, n in ((l1, "l1"), (l1_sf, "l1_sf"), (l2, "l2"), (l2_sf, "l2_sf")):
        _need(t, torch.uint8, n, 3)
    E, twoI, Hh = l1.shape
    H, I = Hh * 2, twoI // 2
    if l1_sf.shape != (E, 2 * I, H // 16) or l2.shape != (E, H, I // 2) or l2_sf.shape != (E, H, I // 16):
        raise ValueError("inconsistent weight shapes")
    n1, n2 = transformed_weight_bytes_nvfp4(E, H, I)
    if out is None:
        l1_t = torch.empty(n1, dtype=torch.uint8, device=l1.device)
        l2_t = torch.empty(n2, dtype=torch.uint8, device=l1.device)
    else:
        l1_t, l2_t = out
        if l1_t.numel() < n1 or l2_t.numel() < n2:
            raise ValueError("output buffers too small")
    _check(load().moe_transform_weights_nvfp4(_ptr(l1), _ptr(l1_sf), _ptr(l2), _ptr(l2_sf), E, H, I,
                                              _ptr(l1_t), _ptr(l2_t), _stream(stream)), "moe_transform_weights_nvfp4")
    return l1_t, l2_t


def transformed_scale_bytes(E: int, H: int, I: int):
    """Byte sizes of the row-major layout's two scale arrays (host-only)."""
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().moe_transformed_scale_bytes(E, H, I, ctypes.byref(a), ctypes.byref(b)),
           "moe_transformed_scale_bytes")
    return a.value, b.value


def transform_scales(l1_sf, l2_sf, out=None, stream=None):
    """[E, 2I, H/32], [E, H, I/32] (u8) -> (l1_sf_t, l2_sf_t) scale-block arrays of
    the row-major layout (u8, 1-D).  ``out`` may give the two destination views."""
    _need(l1_sf, torch.uint8, "l1_sf", 3)
    _need(l2_sf, torch.uint8, "l2_sf", 3)
    E, twoI, Hg = l1_sf.shape
    H, I = Hg * 32, twoI // 2
    if l2_sf.shape != (E, H, I // 32):
        raise ValueError("inconsistent scale shapes")
    n1, n2 = transformed_scale_bytes(E, H, I)
    if out is None:
        a = torch.empty(n1, dtype=torch.uint8, device=l1_sf.device)
        b = torch.empty(n2, dtype=torch.uint8, device=l1_sf.device)
    else:
        a, b = out
        if a.numel() < n1 or b.numel() < n2:
            raise ValueError("output buffers too small")
    _check(load().moe_transform_scales(_ptr(l1_sf), _ptr(l2_sf), E, H, I, _ptr(a), _ptr(b), _stream(stream)),
           "moe_transform_scales")
    return a, b


def workspace_bytes(T: int, E: int, k: int, H: int, I: int) -> int:
    n = ctypes.c_size_t()
    _check(load().moe_workspace_bytes(T, E, k, H, I, ctypes.byref(n)), "moe_workspace_bytes")
    return n.value


def forward_kernel_launches(T: int, E: int, k: int, H: int, I: int) -> int:
    """Kernels one forward call with these sizes enqueues (host-only)."""
    n = ctypes.c_int()
    _check(load().moe_forward_kernel_launches(T, E, k, H, I, ctypes.byref(n)), "moe_forward_kernel_launches")
    return n.value


def forward(x_fp8, x_sf, topk_idx, topk_w, l1_t, l2_t, E: int, H: int, I: int,
            out=None, workspace=None, expert_stats=None, events=None, stream=None, act=None, weights=None):
    """One layer; returns out (bf16 [T, H]).  ``events``: optional list of
    NUM_STAGE_EVENTS torch.cuda.Event recorded at the stage boundaries.
    ``act``: an Activation (see ``activation()``); None = SwiGLU.
    ``weights``: a RowMajorWeights to run the row-major layout (then l1_t and
    l2_t are None); by default l1_t / l2_t are the packet buffers."""
    _need(x_fp8, torch.uint8, "x_fp8", 2)
    _need(x_sf, torch.uint8, "x_sf", 2)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    if weights is None:
        _need(l1_t, torch.uint8, "l1_t")
        _need(l2_t, torch.uint8, "l2_t")
    elif l1_t is not None or l2_t is not None or not isinstance(weights, RowMajorWeights):
        raise ValueError("give either packet buffers l1_t / l2_t or weights=RowMajorWeights(...)")
    T, k = topk_idx.shape
    if x_fp8.shape != (T, H) or x_sf.shape != (T, H // 32) or topk_w.shape != (T, k):
        raise ValueError("inconsistent activation / routing shapes")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x_fp8.device)
    else:
        _need(out, torch.bfloat16, "out", 2)
        if out.shape != (T, H) or out.device != x_fp8.device:
            raise ValueError("out must be bf16 [T, H] on the device of x_fp8")
    if workspace is None:
        workspace = torch.empty(workspace_bytes(T, E, k, H, I), dtype=torch.uint8, device=x_fp8.device)
    else:
        _need(workspace, torch.uint8, "workspace")
    if expert_stats is not None:
        _need(expert_stats, torch.int32, "expert_stats", 1)
    ev = None
    if events is not None:
        if len(events) != NUM_STAGE_EVENTS:
            raise ValueError(f"events must hold {NUM_STAGE_EVENTS} torch.cuda.Event")
        for e in events:
            if e.cuda_event == 0:  # torch creates events lazily, on first record
                e.record(stream if stream is not None else torch.cuda.current_stream())
        ev = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[e.cuda_event for e in events])
    if weights is not None:
        ws_struct = weights.struct()
        st = load().moe_forward_weights(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w),
                                        ctypes.byref(ws_struct), _ptr(out), T, E, k, H, I, _ptr(workspace),
                                        workspace.numel(), _ptr(expert_stats), ev,
                                        ctypes.byref(act) if act is not None else None, _stream(stream))
        _check(st, "moe_forward_weights")
    elif act is None:
        st = load().moe_forward(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(l1_t), _ptr(l2_t),
                                _ptr(out), T, E, k, H, I, _ptr(workspace), workspace.numel(),
                                _ptr(expert_stats), ev, _stream(stream))
        _check(st, "moe_forward")
    else:
        st = load().moe_forward_act(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(l1_t),
                                    _ptr(l2_t), _ptr(out), T, E, k, H, I, _ptr(workspace), workspace.numel(),
                                    _ptr(expert_stats), ev, ctypes.byref(act), _stream(stream))
        _check(st, "moe_forward_act")
    return out


def forward_nvfp4(x_fp4, x_sf, topk_idx, topk_w, l1_t, l2_t, E: int, H: int, I: int,
                  out=None, workspace=None, expert_stats=None, events=None, stream=None, act=None):
    """One layer in NVFP4 (x packed E2M1 [T, H/2] with UE4M3 scales [T, H/16],
    packets from transform_weights_nvfp4); returns out (bf16 [T, H])."""
    _need(x_fp4, torch.uint8, "x_fp4", 2)
    _need(x_sf, torch.uint8, "x_sf", 2)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(l1_t, torch.uint8, "l1_t")
    _need(l2_t, torch.uint8, "l2_t")
    T, k = topk_idx.shape
    if x_fp4.shape != (T, H // 2) or x_sf.shape != (T, H // 16) or topk_w.shape != (T, k):
        raise ValueError("inconsistent activation / routing shapes")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x_fp4.device)
    else:
        _need(out, torch.bfloat16, "out", 2)
        if out.shape != (T, H) or out.device != x_fp4.device:
            raise ValueError("out must be bf16 [T, H] on the device of x_fp4")
    if workspace is None:
        workspace = torch.empty(workspace_bytes(T, E, k, H, I), dtype=torch.uint8, device=x_fp4.device)
    else:
        _need(workspace, torch.uint8, "workspace")
    if expert_stats is not None:
        _need(expert_stats, torch.int32, "expert_stats", 1)
    ev = None
    if events is not None:
        if len(events) != NUM_STAGE_EVENTS:
            raise ValueError(f"events must hold {NUM_STAGE_EVENTS} torch.cuda.Event")
        for e in events:
            if e.cuda_event == 0:
                e.record(stream if stream is not None else torch.cuda.current_stream())
        ev = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[e.cuda_event for e in events])
    st = load().moe_forward_nvfp4(_ptr(x_fp4), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(l1_t), _ptr(l2_t),
                                  _ptr(out), T, E, k, H, I, _ptr(workspace), workspace.numel(), _ptr(expert_stats),
                                  ev, ctypes.byref(act) if act is not None else None, _stream(stream))
    _check(st, "moe_forward_nvfp4")
    return out


def probe_wait_timeout(workspace, timeout_us: int = 1000, stream=None):
    """Diagnostic: a bounded device-side wait that times out (see
    moe_probe_wait_timeout); check_device_error(workspace) then reports it."""
    _need(workspace, torch.uint8, "workspace")
    _check(load().moe_probe_wait_timeout(_ptr(workspace), workspace.numel(), timeout_us, _stream(stream)),
           "moe_probe_wait_timeout")


def shared_workspace_bytes(T_max: int, SH: int, SI: int) -> int:
    """Device workspace bytes of shared_forward for up to T_max tokens."""
    n = ctypes.c_size_t()
    _check(load().moe_shared_workspace_bytes(T_max, SH, SI, ctypes.byref(n)), "moe_shared_workspace_bytes")
    return n.value


def shared_workspace(T_max: int, SH: int, SI: int, device):
    """A zero-filled workspace for shared_forward (the state its first use
    needs; every call leaves it ready for the next)."""
    return torch.zeros(shared_workspace_bytes(T_max, SH, SI), dtype=torch.uint8, device=device)


def shared_forward(x, l1, l2, out=None, workspace=None, act=None, stream=None):
    """The BF16 shared expert: x [T, SH], l1 [2 SI, SH] (gate rows first), l2
    [SH, SI], all bf16; returns y (bf16 [T, SH]).  ``act``: an Activation, None
    = SwiGLU.  ``workspace``: from shared_workspace (zero-filled before its
    first use); None allocates one for this call."""
    _need(x, torch.bfloat16, "x", 2)
    _need(l1, torch.bfloat16, "l1", 2)
    _need(l2, torch.bfloat16, "l2", 2)
    T, SH = x.shape
    SI = l1.shape[0] // 2
    if l1.shape != (2 * SI, SH) or l2.shape != (SH, SI):
        raise ValueError("inconsistent shared-expert shapes")
    if out is None:
        out = torch.empty((T, SH), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, torch.bfloat16, "out", 2)
    if workspace is None:
        workspace = shared_workspace(T, SH, SI, x.device)
    else:
        _need(workspace, torch.uint8, "workspace")
    st = load().moe_shared_forward(_ptr(x), _ptr(l1), _ptr(l2), _ptr(out), T, SH, SI,
                                   ctypes.byref(act) if act is not None else None, _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "moe_shared_forward")
    return out


def forward_static(x_fp8, x_sf, topk_idx, topk_w, l1_t, l2_t, E: int, H: int, I: int,
                   out=None, expert_stats=None, stream=None):
    """The layer for callers that cannot allocate device memory: the scratch is
    the library's fixed STATIC_WORKSPACE_BYTES device array (see
    moe_forward_static in include/moe.h; calls on one device must not overlap
    on the GPU).  ``out`` must be given by such callers; when it is None this
    helper allocates it with torch for convenience."""
    _need(x_fp8, torch.uint8, "x_fp8", 2)
    _need(x_sf, torch.uint8, "x_sf", 2)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(l1_t, torch.uint8, "l1_t")
    _need(l2_t, torch.uint8, "l2_t")
    T, k = topk_idx.shape
    if x_fp8.shape != (T, H) or x_sf.shape != (T, H // 32) or topk_w.shape != (T, k):
        raise ValueError("inconsistent activation / routing shapes")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x_fp8.device)
    else:
        _need(out, torch.bfloat16, "out", 2)
        if out.shape != (T, H) or out.device != x_fp8.device:
            raise ValueError("out must be bf16 [T, H] on the device of x_fp8")
    if expert_stats is not None:
        _need(expert_stats, torch.int32, "expert_stats", 1)
    st = load().moe_forward_static(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), _ptr(topk_w), _ptr(l1_t),
                                   _ptr(l2_t), _ptr(out), T, E, k, H, I, _ptr(expert_stats), None,
                                   _stream(stream))
    _check(st, "moe_forward_static")
    return out


def check_device_error_static(device=None, stream=None) -> int:
    """Synchronises the stream and returns the status the last forward_static
    on ``device`` (a CUDA device or index; default: the current one) left in the
    library's fixed array (0, MOE_ERR_BAD_ROUTING or MOE_ERR_DEVICE_TIMEOUT)."""
    if isinstance(device, int):
        index = device
    else:
        index = None if device is None else torch.device(device).index
        if index is None:
            index = torch.cuda.current_device()
    return load().moe_check_device_error_static(int(index), _stream(stream))


def read_routing(workspace, T: int, E: int, k: int, H: int, I: int, stream=None):
    """Routing metadata of the last forward on ``workspace`` (host int32 tensors)."""
    count = torch.empty(E, dtype=torch.int32)
    offset = torch.empty(E + 1, dtype=torch.int32)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32)
    inv = torch.empty(max(T * k, 1), dtype=torch.int32)
    _check(load().moe_read_routing(_ptr(workspace), T, E, k, H, I, _ptr(count), _ptr(offset), _ptr(perm),
                                   _ptr(inv), _stream(stream)), "moe_read_routing")
    n = int(offset[E])
    return dict(count=count, offset=offset, perm=perm[:n].clone(), inv=inv[: T * k].clone())


def check_device_error(workspace, stream=None) -> int:
    """Synchronises the stream and returns the status of the last forward on
    ``workspace`` (0, MOE_ERR_BAD_ROUTING or MOE_ERR_DEVICE_TIMEOUT)."""
    return load().moe_check_device_error(_ptr(workspace), _stream(stream))


class MoELayer:
    """Holds one layer's transformed weights and a workspace for up to T_max tokens."""

    def __init__(self, l1_t, l2_t, E: int, k: int, H: int, I: int, T_max: int, device=None, weights=None,
                 fmt: str = "mx"):
        if fmt not in ("mx", "nvfp4") or (fmt == "nvfp4" and weights is not None):
            raise ValueError("fmt is 'mx' or 'nvfp4' (NVFP4 takes packet buffers)")
        self.l1_t, self.l2_t, self.weights, self.fmt = l1_t, l2_t, weights, fmt
        self.E, self.k, self.H, self.I, self.T_max = E, k, H, I, T_max
        device = device or (l1_t.device if weights is None else weights.l1.device)
        self.workspace = torch.empty(workspace_bytes(T_max, E, k, H, I), dtype=torch.uint8, device=device)

    def __call__(self, x_fp8, x_sf, topk_idx, topk_w, out=None, expert_stats=None, events=None, stream=None,
                 act=None):
        if topk_idx.shape[0] > self.T_max:
            raise ValueError(f"T={topk_idx.shape[0]} exceeds T_max={self.T_max}")
        if self.fmt == "nvfp4":
            return forward_nvfp4(x_fp8, x_sf, topk_idx, topk_w, self.l1_t, self.l2_t, self.E, self.H, self.I,
                                 out=out, workspace=self.workspace, expert_stats=expert_stats, events=events,
                                 stream=stream, act=act)
        return forward(x_fp8, x_sf, topk_idx, topk_w, self.l1_t, self.l2_t, self.E, self.H, self.I,
                       out=out, workspace=self.workspace, expert_stats=expert_stats, events=events,
                       stream=stream, act=act, weights=self.weights)


# ------------------------------------------------------------ expert parallelism
def ep_workspace_bytes(T: int, E: int, k: int, H: int) -> int:
    """Bytes of the dispatch workspace for up to T tokens (host-only)."""
    n = ctypes.c_size_t()
    _check(load().moe_ep_workspace_bytes(T, E, k, H, ctypes.byref(n)), "moe_ep_workspace_bytes")
    return n.value


def ep_dispatch(x_fp8, x_sf, topk_idx, E: int, ranks: int, workspace, send_x=None, send_sf=None, send_eid=None,
                send_counts=None, stream=None):
    """Routing and the send buffers of expert parallelism: returns (send_x u8
    [T*k, H], send_sf u8 [T*k, H/32], send_eid i64 [T*k], send_counts i64
    [ranks]); the first sum(send_counts) rows, grouped by destination rank,
    are written.  ``workspace`` (u8, ep_workspace_bytes) must stay untouched
    until the matching ep_combine."""
    _need(x_fp8, torch.uint8, "x_fp8", 2)
    _need(x_sf, torch.uint8, "x_sf", 2)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(workspace, torch.uint8, "workspace")
    T, H = x_fp8.shape
    k = topk_idx.shape[1]
    if x_sf.shape != (T, H // 32) or topk_idx.shape[0] != T:
        raise ValueError("inconsistent input shapes")
    dev = x_fp8.device
    if send_x is None:
        send_x = torch.empty((T * k, H), dtype=torch.uint8, device=dev)
    if send_sf is None:
        send_sf = torch.empty((T * k, H // 32), dtype=torch.uint8, device=dev)
    if send_eid is None:
        send_eid = torch.empty(T * k, dtype=torch.int64, device=dev)
    if send_counts is None:
        send_counts = torch.empty(ranks, dtype=torch.int64, device=dev)
    _need(send_x, torch.uint8, "send_x", 2)
    _need(send_sf, torch.uint8, "send_sf", 2)
    _need(send_eid, torch.int64, "send_eid", 1)
    _need(send_counts, torch.int64, "send_counts", 1)
    if (send_x.shape[0] < T * k or send_x.shape[1] != H or send_sf.shape[0] < T * k or send_sf.shape[1] != H // 32
            or send_eid.numel() < T * k or send_counts.numel() != ranks):
        raise ValueError("send buffers too small")
    _check(load().moe_ep_dispatch(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), T, E, k, H, ranks, _ptr(workspace),
                                  workspace.numel(), _ptr(send_x), _ptr(send_sf), _ptr(send_eid), _ptr(send_counts),
                                  _stream(stream)), "moe_ep_dispatch")
    return send_x, send_sf, send_eid, send_counts


def ep_combine(y, topk_w, E: int, workspace, out=None, stream=None):
    """out (bf16 [T, H]) = the top-k-weighted sum of the returned rows y (bf16
    [n, H], in send order) through the inverse permutation of the ep_dispatch
    that used ``workspace`` with the same T, E, k, H."""
    _need(y, torch.bfloat16, "y", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(workspace, torch.uint8, "workspace")
    T, k = topk_w.shape
    H = y.shape[1]
    if y.shape[0] < T * k:
        # the combine reads row inv[t*k + j] of y, and inv reaches T*k - 1
        raise ValueError("y must hold at least T*k rows (the dispatch's routed rows)")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=topk_w.device)
    _need(out, torch.bfloat16, "out", 2)
    if out.shape != (T, H):
        raise ValueError("out must be [T, H]")
    _check(load().moe_ep_combine(_ptr(y), _ptr(topk_w), T, E, k, H, _ptr(workspace), workspace.numel(), _ptr(out),
                                 _stream(stream)), "moe_ep_combine")
    return out


def ep_combine_peers(peer_y, recv_base, topk_idx, topk_w, E: int, H: int, workspace, out=None, stream=None):
    """The combine reading each returned row from the rank that computed it:
    ``peer_y`` i64 [ranks] device tensor of the ranks' output addresses (bf16
    [rows, H] each, mapped into this process), ``recv_base`` i64 [ranks]
    device tensor (where this rank's rows start in each rank's received
    rows); returns out (bf16 [T, H]).  The peers' buffers are raw addresses
    that this function cannot size-check: rank r's must hold at least
    recv_base[r] + (rows this rank sent to r) rows."""
    _need(peer_y, torch.int64, "peer_y", 1)
    _need(recv_base, torch.int64, "recv_base", 1)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(workspace, torch.uint8, "workspace")
    T, k = topk_w.shape
    ranks = peer_y.numel()
    if recv_base.numel() != ranks or topk_idx.shape != (T, k):
        raise ValueError("inconsistent shapes")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=topk_w.device)
    _need(out, torch.bfloat16, "out", 2)
    if out.shape != (T, H):
        raise ValueError("out must be [T, H]")
    _check(load().moe_ep_combine_peers(_ptr(peer_y), _ptr(recv_base), _ptr(topk_idx), _ptr(topk_w), T, E, k, H,
                                       ranks, _ptr(workspace), workspace.numel(), _ptr(out), _stream(stream)),
           "moe_ep_combine_peers")
    return out


def ep_route(topk_idx, E: int, H: int, ranks: int, workspace, send_counts=None, stream=None):
    """The dispatch's routing and per-rank row counts without copying rows
    (for ep_dispatch_peers); returns send_counts (i64 [ranks], device)."""
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(workspace, torch.uint8, "workspace")
    T, k = topk_idx.shape
    if send_counts is None:
        send_counts = torch.empty(ranks, dtype=torch.int64, device=workspace.device)
    _need(send_counts, torch.int64, "send_counts", 1)
    if send_counts.numel() != ranks:
        raise ValueError("send_counts must hold one count per rank")
    _check(load().moe_ep_route(_ptr(topk_idx), T, E, k, H, ranks, _ptr(workspace), workspace.numel(),
                               _ptr(send_counts), _stream(stream)), "moe_ep_route")
    return send_counts


def ep_dispatch_peers(x_fp8, x_sf, topk_idx, E: int, workspace, peer_x, peer_sf, peer_eid, recv_base, stream=None):
    """Writes this rank's routed rows into the ranks' receive buffers (after
    ep_route on the same workspace): ``peer_x`` / ``peer_sf`` / ``peer_eid``
    i64 [ranks] device tensors of the buffers' addresses, ``recv_base`` i64
    [ranks] device tensor of this rank's first row in each of them."""
    _need(x_fp8, torch.uint8, "x_fp8", 2)
    _need(x_sf, torch.uint8, "x_sf", 2)
    _need(topk_idx, torch.int64, "topk_idx", 2)
    _need(workspace, torch.uint8, "workspace")
    for t, n in ((peer_x, "peer_x"), (peer_sf, "peer_sf"), (peer_eid, "peer_eid"), (recv_base, "recv_base")):
        _need(t, torch.int64, n, 1)
    T, H = x_fp8.shape
    k = topk_idx.shape[1]
    ranks = peer_x.numel()
    if x_sf.shape != (T, H // 32) or topk_idx.shape[0] != T or not (
            peer_sf.numel() == peer_eid.numel() == recv_base.numel() == ranks):
        raise ValueError("inconsistent shapes")
    _check(load().moe_ep_dispatch_peers(_ptr(x_fp8), _ptr(x_sf), _ptr(topk_idx), T, E, k, H, ranks, _ptr(workspace),
                                        workspace.numel(), _ptr(peer_x), _ptr(peer_sf), _ptr(peer_eid),
                                        _ptr(recv_base), _stream(stream)), "moe_ep_dispatch_peers")


# ------------------------------------------------------------ peer buffers (CUDA IPC)
def ipc_handle(t: torch.Tensor):
    """(handle bytes, byte offset) of device tensor t's allocation, for
    another process's ipc_open (moe_ipc_handle)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("ipc_handle takes a CUDA tensor")
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_size_t()
    _check(load().moe_ipc_handle(_ptr(t), buf, ctypes.byref(off)), "moe_ipc_handle")
    return buf.raw, off.value


def ipc_open(handle: bytes, device: int) -> int:
    """Maps another process's allocation into this one on CUDA device
    ``device``; returns the mapped base address (moe_ipc_open)."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has IPC_HANDLE_BYTES bytes")
    base = ctypes.c_void_p()
    _check(load().moe_ipc_open(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES), int(device),
                               ctypes.byref(base)), "moe_ipc_open")
    return int(base.value)


def ipc_close(base: int) -> None:
    """Unmaps a base returned by ipc_open (moe_ipc_close)."""
    _check(load().moe_ipc_close(ctypes.c_void_p(base)), "moe_ipc_close")
