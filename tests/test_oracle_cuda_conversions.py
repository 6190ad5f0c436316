"""Pins for the oracle's FP8 E4M3 / FP4 E2M1 decoders and its
round-to-nearest-even rule against CUDA's own conversions (cuda_fp8.h,
cuda_fp4.h: `__nv_cvt_fp8_to_halfraw`, `__nv_cvt_fp4_to_halfraw`,
`__nv_cvt_float_to_fp8` with satfinite, `__nv_cvt_float_to_fp4` with
cudaRoundNearest), called through the test-only wrapper
`cuda_conversions.cu`: on the host (runs here) and in a kernel on the GPU.
On the host also: the UE8M0 scale rule against `__nv_cvt_double_to_e8m0`
rounding toward +infinity, the UE8M0 decoder against
`__nv_cvt_e8m0_to_bf16raw`, and the bf16 rounding against
`__float2bfloat16_rn`.

The inputs cover every code, a dense grid over each format's range, every
midpoint between adjacent codes (where ties-to-even decides) and random
values; codes must agree exactly, the sign of zero included.
"""
import ctypes

import numpy as np
import pytest

import cuda_conversions as cc
import oracle

F32P, U8P = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_uint8)


@pytest.fixture(scope="module")
def cvt():
    return cc.load()


def _oracle_values(decode, n):
    return np.array([decode(c) for c in range(n)])


def _positive_codes(n_codes, decode):
    v = _oracle_values(decode, n_codes)
    half = v[: n_codes // 2]
    return np.array(sorted(set(half[np.isfinite(half)].tolist())))


def e4m3_inputs():
    """Values with |v| <= 448 (the range the quantiser feeds in)."""
    pos = _positive_codes(256, oracle.e4m3_value)
    mids = (pos[1:] + pos[:-1]) / 2                   # ties, exact in fp32
    quarter = (3 * pos[1:] + pos[:-1]) / 4            # just off the ties
    grid = np.arange(-448 * 64, 448 * 64 + 1) / 64    # the normal range, step 1/64
    tiny = np.ldexp(np.arange(-4096, 4097), -16)      # the subnormal binade, step 2^-16
    rnd = np.random.default_rng(8).uniform(-448.0, 448.0, 20000)
    v = np.concatenate([pos, mids, quarter, grid, tiny, rnd])
    return np.concatenate([v, -v]).astype(np.float32)


def e2m1_inputs():
    """Values with |v| <= 6."""
    pos = _positive_codes(16, oracle.e2m1_value)
    mids = (pos[1:] + pos[:-1]) / 2
    grid = np.arange(-6 * 1024, 6 * 1024 + 1) / 1024
    rnd = np.random.default_rng(4).uniform(-6.0, 6.0, 20000)
    v = np.concatenate([pos, mids, grid, rnd])
    return np.concatenate([v, -v]).astype(np.float32)


def _oracle_codes(vals, rnd):
    return np.array([rnd(float(x)) for x in vals], dtype=np.uint8)


def _check_decode(got, n, decode):
    ref = _oracle_values(decode, n)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].astype(np.float64), ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ------------------------------------------------------------- host path
def test_decode_all_codes_match_cuda_host(cvt):
    d8 = np.zeros(256, np.float32)
    assert cvt.cvt_host_decode_e4m3(d8.ctypes.data_as(F32P)) == 0
    _check_decode(d8, 256, oracle.e4m3_value)
    d4 = np.zeros(16, np.float32)
    assert cvt.cvt_host_decode_e2m1(d4.ctypes.data_as(F32P)) == 0
    _check_decode(d4, 16, oracle.e2m1_value)


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_rounding_matches_cuda_host(cvt, fmt):
    vals = e4m3_inputs() if fmt == "e4m3" else e2m1_inputs()
    got = np.zeros(len(vals), np.uint8)
    fn = cvt.cvt_host_round_e4m3 if fmt == "e4m3" else cvt.cvt_host_round_e2m1
    assert fn(vals.ctypes.data_as(F32P), got.ctypes.data_as(U8P), len(vals)) == 0
    ref = _oracle_codes(vals, oracle.round_e4m3 if fmt == "e4m3" else oracle.round_e2m1)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{fmt}: {vals[bad[:8]]} -> cuda {got[bad[:8]]}, oracle {ref[bad[:8]]}"


def _amax_values():
    """Positive fp32 magnitudes over the whole exponent range, subnormals
    included, plus every boundary Q * 2^e of both formats and its fp32
    neighbours (where the rounding up changes)."""
    rng = np.random.default_rng(11)
    v = [np.ldexp(rng.uniform(1.0, 2.0, 20000), rng.integers(-149, 128, 20000)),
         np.ldexp(1.0, np.arange(-149, 128)), [np.finfo(np.float32).max, np.finfo(np.float32).tiny]]
    for q in (448.0, 6.0):
        b = np.ldexp(q, np.arange(-160, 128))
        b = b[b < np.finfo(np.float32).max].astype(np.float32)
        v += [b, np.nextafter(b, np.float32(np.inf)), np.nextafter(b, np.float32(0))]
    a = np.concatenate([np.asarray(x, np.float64).ravel() for x in v]).astype(np.float32)
    return np.unique(a[np.isfinite(a) & (a > 0)])


@pytest.mark.parametrize("qmax", [448.0, 6.0], ids=["e4m3", "e2m1"])
def test_scale_rule_matches_cuda_e8m0_round_up(cvt, qmax):
    """b = e + 127, e the smallest integer with amax <= qmax * 2^e (clamped to
    [0, 254]), is CUDA's UE8M0 of amax / qmax rounded up to a power of two
    (clipped to 2^-127 .. 2^127).  The double quotient of an fp32 amax by 448
    = 7 * 2^6 or 6 = 3 * 2 lands on a power of two only where the exact one
    does, so the library call sees the exact case split.  (amax = 0 is the
    oracle's own reading, scale 1, and is not compared.)"""
    # fp32 magnitudes, and a few doubles beyond fp32's range for the upper clamp
    amax = np.concatenate([_amax_values().astype(np.float64), [1e39, 1e100, 1e300]])
    ratio = amax / qmax
    got = np.zeros(len(amax), np.uint8)
    assert cvt.cvt_host_e8m0_ceil(ratio.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                  got.ctypes.data_as(U8P), len(amax)) == 0
    ref = np.array([min(max(oracle.scale_exponent(float(a), qmax) + 127, 0), 254) for a in amax], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"amax {amax[bad[:6]]}: cuda {got[bad[:6]]}, oracle {ref[bad[:6]]}"
    assert ref[0] == 0 and ref[-1] == 254   # both clamps reached


def test_ue8m0_decode_matches_cuda(cvt):
    d = np.zeros(256, np.float32)
    assert cvt.cvt_host_decode_e8m0(d.ctypes.data_as(F32P)) == 0
    ref = np.array([oracle.ue8m0_value(b) for b in range(256)])
    assert np.isnan(d[255]) and np.isnan(ref[255])
    assert np.array_equal(d[:255].astype(np.float64), ref[:255])


def test_bf16_rounding_matches_cuda(cvt):
    """Random fp32 bit patterns (every exponent, subnormals, infinities), the
    exact ties between two bf16 values with even and odd last bits, and
    their fp32 neighbours; NaN only by class (the oracle writes one
    canonical NaN)."""
    rng = np.random.default_rng(16)
    bits = [rng.integers(0, 1 << 32, 60000, dtype=np.uint64).astype(np.uint32)]
    hi = rng.integers(0, 1 << 16, 8000, dtype=np.uint64).astype(np.uint32) << 16
    bits += [hi | 0x8000, hi | 0x7FFF, hi | 0x8001, np.array([0x7F800000, 0xFF800000, 0, 0x80000000], np.uint32)]
    x = np.concatenate(bits).view(np.float32)
    got = np.zeros(len(x), np.uint16)
    assert cvt.cvt_host_f32_to_bf16(x.ctypes.data_as(F32P), got.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)),
                                    len(x)) == 0
    ref = oracle.f32_to_bf16(x)
    nan = np.isnan(x)
    assert np.all((got[nan] & 0x7F80) == 0x7F80) and np.all(got[nan] & 0x7F)
    bad = np.nonzero((got != ref) & ~nan)[0]
    assert bad.size == 0, f"{x[bad[:6]]}: cuda {got[bad[:6]]}, oracle {ref[bad[:6]]}"


def test_bad_arguments_are_refused(cvt):
    assert cvt.cvt_host_decode_e4m3(None) == -1
    assert cvt.cvt_host_round_e2m1(None, None, -1) == -1
    assert cvt.cvt_host_round_e4m3(None, None, 0) == 0


# ------------------------------------------------------------ device path
@pytest.mark.gpu
def test_decode_all_codes_match_cuda_device(cvt):
    import torch
    s = torch.cuda.current_stream().cuda_stream
    d8 = torch.empty(256, dtype=torch.float32, device="cuda")
    d4 = torch.empty(16, dtype=torch.float32, device="cuda")
    assert cvt.cvt_dev_decode_e4m3(d8.data_ptr(), s) == 0
    assert cvt.cvt_dev_decode_e2m1(d4.data_ptr(), s) == 0
    torch.cuda.synchronize()
    _check_decode(d8.cpu().numpy(), 256, oracle.e4m3_value)
    _check_decode(d4.cpu().numpy(), 16, oracle.e2m1_value)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_rounding_matches_cuda_device(cvt, fmt):
    import torch
    vals = e4m3_inputs() if fmt == "e4m3" else e2m1_inputs()
    x = torch.from_numpy(vals).cuda()
    y = torch.empty(len(vals), dtype=torch.uint8, device="cuda")
    fn = cvt.cvt_dev_round_e4m3 if fmt == "e4m3" else cvt.cvt_dev_round_e2m1
    assert fn(x.data_ptr(), y.data_ptr(), len(vals), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    ref = _oracle_codes(vals, oracle.round_e4m3 if fmt == "e4m3" else oracle.round_e2m1)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{fmt}: {vals[bad[:8]]} -> cuda {got[bad[:8]]}, oracle {ref[bad[:8]]}"
