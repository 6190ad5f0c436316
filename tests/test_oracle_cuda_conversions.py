"""Pins for the oracle's FP8 E4M3 / FP4 E2M1 decoders and its
round-to-nearest-even rule against CUDA's own conversions (cuda_fp8.h,
cuda_fp4.h: `__nv_cvt_fp8_to_halfraw`, `__nv_cvt_fp4_to_halfraw`,
`__nv_cvt_float_to_fp8` with satfinite, `__nv_cvt_float_to_fp4` with
cudaRoundNearest), called through the test-only wrapper
`cuda_conversions.cu`: on the host (runs here) and in a kernel on the GPU.

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
