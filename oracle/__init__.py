"""CPU oracle of the FP8 x FP4 MoE expert layer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference leg may import this package.  The CUDA library never calls it and
shares no code with it.  The arithmetic lives in ``moe_oracle.c`` (plain C,
built with gcc into ``libmoe_oracle.so`` next to it); this module only
marshals numpy arrays.

Parity status of each function (the pins are the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py``):

* ``e4m3_value`` / ``e2m1_value`` / ``ue8m0_value``: pinned against torch's
  float8 conversions and the OCP MX element tables.
* ``quantize_e4m3`` / ``quantize_e2m1``: pinned against exact rational
  evaluation of 2^ceil(log2(amax/Q)), torch's RNE float8 cast and a
  brute-force nearest-value search.
* ``route``: pinned against numpy's stable argsort and routing invariants.
* ``forward``: pinned against a float64 numpy evaluation of every selected
  expert on tiny inputs, the dense single-expert special case and layer
  invariants (token-permutation equivariance, identical experts, determinism).
* ``shared_forward`` (the BF16 shared expert): pinned against a float64 numpy
  evaluation with torch's bf16 rounding between the steps, the dense identity
  special case and token-permutation equivariance.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def build(force: bool = False, out: str | None = None, extra_flags=()) -> str:
    """Compile moe_oracle.c with gcc.  Returns the path of the shared library."""
    out = out or _LIB
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    cmd = ["gcc", "-O2", "-std=gnu11", "-fno-fast-math", "-ffp-contract=off", "-Wall",
           "-shared", "-fPIC", "-pthread", *extra_flags, "-o", out + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _declare(lib):
    c = ctypes
    P = c.c_void_p
    lib.oracle_e4m3_value.restype = c.c_double
    lib.oracle_e4m3_value.argtypes = [c.c_uint32]
    lib.oracle_e2m1_value.restype = c.c_double
    lib.oracle_e2m1_value.argtypes = [c.c_uint32]
    lib.oracle_ue8m0_value.restype = c.c_double
    lib.oracle_ue8m0_value.argtypes = [c.c_uint32]
    lib.oracle_scale_exponent.restype = c.c_int
    lib.oracle_scale_exponent.argtypes = [c.c_double, c.c_double]
    lib.oracle_round_e4m3.restype = c.c_uint32
    lib.oracle_round_e4m3.argtypes = [c.c_double]
    lib.oracle_round_e2m1.restype = c.c_uint32
    lib.oracle_round_e2m1.argtypes = [c.c_double]
    lib.oracle_quantize_e4m3.restype = None
    lib.oracle_quantize_e4m3.argtypes = [P, c.c_int64, c.c_int64, P, P]
    lib.oracle_quantize_e2m1.restype = None
    lib.oracle_quantize_e2m1.argtypes = [P, c.c_int64, c.c_int64, P, P]
    lib.oracle_f32_to_bf16.restype = c.c_uint16
    lib.oracle_f32_to_bf16.argtypes = [c.c_float]
    lib.oracle_route.restype = c.c_int
    lib.oracle_route.argtypes = [P, c.c_int, c.c_int, c.c_int, P, P, P, P]
    lib.oracle_num_threads.restype = c.c_int
    lib.oracle_num_threads.argtypes = [c.c_int]
    lib.oracle_moe_forward_act.restype = c.c_int
    lib.oracle_moe_forward_act.argtypes = [P, P, P, P, P, P, P, P,
                                           c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                           P, c.c_int, c.c_int, c.c_int,
                                           c.c_int, c.c_double, c.c_double,
                                           P, P, P, P, P, P]
    lib.oracle_moe_forward_fmt.restype = c.c_int
    lib.oracle_moe_forward_fmt.argtypes = [P, P, P, P, P, P, P, P,
                                           c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                           P, c.c_int, c.c_int, c.c_int,
                                           c.c_int, c.c_double, c.c_double, c.c_int,
                                           P, P, P, P, P, P]
    lib.oracle_ue4m3_value.restype = c.c_double
    lib.oracle_ue4m3_value.argtypes = [c.c_uint32]
    lib.oracle_nvfp4_scale.restype = c.c_uint32
    lib.oracle_nvfp4_scale.argtypes = [c.c_double]
    lib.oracle_quantize_nvfp4.restype = None
    lib.oracle_quantize_nvfp4.argtypes = [P, c.c_int64, c.c_int64, P, P]
    lib.oracle_shared_forward.restype = c.c_int
    lib.oracle_shared_forward.argtypes = [P, P, P, c.c_int, c.c_int, c.c_int, P, c.c_int, c.c_int,
                                          c.c_int, c.c_double, c.c_double, P, P]
    lib.oracle_moe_forward.restype = c.c_int
    lib.oracle_moe_forward.argtypes = [P, P, P, P, P, P, P, P,
                                       c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                       P, c.c_int, c.c_int, c.c_int,
                                       P, P, P, P, P, P]
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library.  With ``path`` a
    separately built copy is loaded and returned without caching."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


# ---------------------------------------------------------------- decoders
def e4m3_value(code: int, lib=None) -> float:
    return (lib or load()).oracle_e4m3_value(code)


def e2m1_value(code: int, lib=None) -> float:
    return (lib or load()).oracle_e2m1_value(code)


def ue8m0_value(b: int, lib=None) -> float:
    return (lib or load()).oracle_ue8m0_value(b)


def scale_exponent(amax: float, qmax: float, lib=None) -> int:
    return (lib or load()).oracle_scale_exponent(amax, qmax)


def round_e4m3(v: float, lib=None) -> int:
    return (lib or load()).oracle_round_e4m3(v)


def round_e2m1(v: float, lib=None) -> int:
    return (lib or load()).oracle_round_e2m1(v)


def f32_to_bf16(a, lib=None) -> np.ndarray:
    lib = lib or load()
    a = np.asarray(a, dtype=np.float32)
    return np.array([lib.oracle_f32_to_bf16(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


# ---------------------------------------------------------------- quantisers
def quantize_e4m3(src, lib=None):
    """fp32 [rows, cols] -> (codes u8 [rows, cols], sf u8 [rows, cols/32])."""
    lib = lib or load()
    src = _c(src, np.float32)
    rows, cols = src.shape
    assert cols % 32 == 0
    codes = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 32), np.uint8)
    lib.oracle_quantize_e4m3(_ptr(src), rows, cols, _ptr(codes), _ptr(sf))
    return codes, sf


def quantize_e2m1(src, lib=None):
    """fp32 [rows, cols] -> (packed u8 [rows, cols/2] (even element in the low
    nibble), sf u8 [rows, cols/32])."""
    lib = lib or load()
    src = _c(src, np.float32)
    rows, cols = src.shape
    assert cols % 32 == 0
    packed = np.empty((rows, cols // 2), np.uint8)
    sf = np.empty((rows, cols // 32), np.uint8)
    lib.oracle_quantize_e2m1(_ptr(src), rows, cols, _ptr(packed), _ptr(sf))
    return packed, sf


def ue4m3_value(b: int, lib=None) -> float:
    return (lib or load()).oracle_ue4m3_value(b)


def nvfp4_scale(amax: float, lib=None) -> int:
    """UE4M3 scale code of a 16-element NVFP4 group with this amax."""
    return (lib or load()).oracle_nvfp4_scale(amax)


def quantize_nvfp4(src, lib=None):
    """fp32 [rows, cols] -> (packed E2M1 u8 [rows, cols/2] (even element in the
    low nibble), UE4M3 scale bytes u8 [rows, cols/16])."""
    lib = lib or load()
    src = _c(src, np.float32)
    rows, cols = src.shape
    assert cols % 16 == 0
    packed = np.empty((rows, cols // 2), np.uint8)
    sf = np.empty((rows, cols // 16), np.uint8)
    lib.oracle_quantize_nvfp4(_ptr(src), rows, cols, _ptr(packed), _ptr(sf))
    return packed, sf


# ---------------------------------------------------------------- routing
def route(topk_idx, E: int, lib=None):
    """Stable per-expert permutation.  Returns dict(count, offset, perm, inv,
    dropped); ``perm`` holds the sum(count) valid entries."""
    lib = lib or load()
    idx = _c(topk_idx, np.int64)
    T, k = idx.shape
    count = np.empty(E, np.int32)
    offset = np.empty(E + 1, np.int32)
    perm = np.full(max(T * k, 1), -1, np.int32)
    inv = np.empty(max(T * k, 1), np.int32)
    dropped = lib.oracle_route(_ptr(idx), T, k, E, _ptr(count), _ptr(offset), _ptr(perm), _ptr(inv))
    n = int(count.sum())
    return dict(count=count, offset=offset, perm=perm[:n].copy(), inv=inv[: T * k].copy(), dropped=dropped)


# ---------------------------------------------------------------- layer
def forward(x_codes, x_sf, topk_idx, topk_w, experts: dict, E: int, H: int, I: int,
            tokens=None, precision: str = "fp32", threads: int = 0,
            intermediates: bool = False, activation: str = "swiglu", beta: float = 1.0,
            linear_beta=None, fmt: str = "mx", lib=None):
    """Evaluate the layer for the listed tokens (all when ``tokens`` is None).

    ``experts`` maps expert id -> (l1 [2I, H/2] u8, l1_sf [2I, H/32] u8,
    l2 [H, I/2] u8, l2_sf [H, I/32] u8); every expert a listed token uses must
    be present.  Returns dict with ``out_bf16`` (uint16 bits, [ntok, H]) and
    ``out_f32``; with ``intermediates`` also ``h_pre`` [ntok, k, I] (the
    activation before requantisation), ``h_q``, ``h_sf`` and ``y`` [ntok, k, H].
    ``activation``: "swiglu" or "situ" (with ``beta`` and optional
    ``linear_beta``).  ``fmt``: "mx" (the above) or "nvfp4": x packed E2M1
    [T, H/2] with UE4M3 scales [T, H/16], the experts' scales [.., K/16]
    UE4M3, h requantised to NVFP4 (``h_q`` [ntok, k, I/2], ``h_sf`` [.., I/16]).
    """
    lib = lib or load()
    x_codes = _c(x_codes, np.uint8)
    x_sf = _c(x_sf, np.uint8)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_w, np.float32)
    T, k = idx.shape
    nv = {"mx": 0, "nvfp4": 1}[fmt]
    gs = 16 if nv else 32
    xcols = H // 2 if nv else H
    assert x_codes.shape == (T, xcols) and x_sf.shape == (T, H // gs) and w.shape == (T, k)
    if tokens is None:
        tok = None
        ntok = T
    else:
        tok = _c(tokens, np.int32)
        ntok = int(tok.size)
    keep = []
    arrs = [(ctypes.c_void_p * E)() for _ in range(4)]
    for e, mats in experts.items():
        shapes = [(2 * I, H // 2), (2 * I, H // gs), (H, I // 2), (H, I // gs)]
        for a, m, shp in zip(arrs, mats, shapes):
            m = _c(m, np.uint8)
            assert m.shape == shp, (m.shape, shp)
            keep.append(m)
            a[e] = m.ctypes.data
    out_bf16 = np.empty((ntok, H), np.uint16)
    out_f32 = np.empty((ntok, H), np.float32)
    h_pre = np.empty((ntok, k, I), np.float32) if intermediates else None
    h_q = np.empty((ntok, k, I // 2 if nv else I), np.uint8) if intermediates else None
    h_sf = np.empty((ntok, k, I // gs), np.uint8) if intermediates else None
    y = np.empty((ntok, k, H), np.float32) if intermediates else None
    act = {"swiglu": 0, "situ": 1}[activation]
    rc = lib.oracle_moe_forward_fmt(
        _ptr(x_codes), _ptr(x_sf), _ptr(idx), _ptr(w),
        ctypes.cast(arrs[0], ctypes.c_void_p), ctypes.cast(arrs[1], ctypes.c_void_p),
        ctypes.cast(arrs[2], ctypes.c_void_p), ctypes.cast(arrs[3], ctypes.c_void_p),
        T, E, k, H, I, _ptr(tok), ntok, 1 if precision == "double" else 0, threads,
        act, float(beta), float(linear_beta or 0.0), nv,
        _ptr(out_bf16), _ptr(out_f32), _ptr(h_pre), _ptr(h_q), _ptr(h_sf), _ptr(y))
    if rc == -1:
        raise KeyError("a listed token routes to an expert whose weights were not given")
    if rc != 0:
        raise ValueError(f"oracle_moe_forward rejected its arguments (rc={rc})")
    res = dict(out_bf16=out_bf16, out_f32=out_f32)
    if intermediates:
        res.update(h_pre=h_pre, h_q=h_q, h_sf=h_sf, y=y)
    return res


def shared_forward(x_bits, l1_bits, l2_bits, tokens=None, activation: str = "swiglu", beta: float = 1.0,
                   linear_beta=None, threads: int = 0, intermediates: bool = False, lib=None):
    """The BF16 shared expert (bf16 bit patterns as uint16): x [T, SH], l1
    [2 SI, SH] (gate rows first), l2 [SH, SI].  Returns dict with ``y`` [ntok,
    SH] (bf16 bits) and, with ``intermediates``, ``h`` [ntok, SI] (the rounded
    activation)."""
    lib = lib or load()
    x = _c(x_bits, np.uint16)
    l1 = _c(l1_bits, np.uint16)
    l2 = _c(l2_bits, np.uint16)
    T, SH = x.shape
    SI = l1.shape[0] // 2
    assert l1.shape == (2 * SI, SH) and l2.shape == (SH, SI)
    if tokens is None:
        tok, ntok = None, T
    else:
        tok = _c(tokens, np.int32)
        ntok = int(tok.size)
    y = np.empty((ntok, SH), np.uint16)
    h = np.empty((ntok, SI), np.uint16) if intermediates else None
    act = {"swiglu": 0, "situ": 1}[activation]
    rc = lib.oracle_shared_forward(_ptr(x), _ptr(l1), _ptr(l2), T, SH, SI, _ptr(tok), ntok, threads, act,
                                   float(beta), float(linear_beta or 0.0), _ptr(y), _ptr(h))
    if rc != 0:
        raise ValueError(f"oracle_shared_forward rejected its arguments (rc={rc})")
    res = dict(y=y)
    if intermediates:
        res["h"] = h
    return res


def num_threads(requested: int = 0, lib=None) -> int:
    return (lib or load()).oracle_num_threads(requested)


def bf16_bits_to_f32(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- inputs
def quantize_inputs(x_bf16_f32, l1_f32: dict, l2_f32: dict, fmt: str = "mx", lib=None):
    """Quantise fp32 copies of the bf16 draws: x -> E4M3, expert weights -> E2M1
    (fmt "mx"), or all to NVFP4 (fmt "nvfp4").  Returns (x_codes, x_sf,
    experts) in the layout ``forward`` takes."""
    qx, qw = (quantize_nvfp4, quantize_nvfp4) if fmt == "nvfp4" else (quantize_e4m3, quantize_e2m1)
    xq, xs = qx(x_bf16_f32, lib)
    experts = {}
    for e in l1_f32:
        a, b = qw(l1_f32[e], lib)
        c, d = qw(l2_f32[e], lib)
        experts[e] = (a, b, c, d)
    return xq, xs, experts
