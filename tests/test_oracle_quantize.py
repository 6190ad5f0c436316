"""Pins for the oracle's quantisation rule: per row, per 32 elements,
scale = 2^ceil(log2(amax/Q)) as a UE8M0 byte, codes = RNE(v / scale).

Independent references: exact rational arithmetic (fractions) for the scale
exponent, torch's RNE float8_e4m3fn cast, a brute-force nearest-value search
for E2M1, torch's bfloat16 cast for the output rounding.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def exact_exponent(amax: float, q: int) -> int:
    """Smallest integer e with amax <= q * 2^e, in exact rationals."""
    a = Fraction(amax)
    e = 0
    while a > q * Fraction(2) ** e:
        e += 1
    while a <= q * Fraction(2) ** (e - 1):
        e -= 1
    return e


@pytest.mark.parametrize("q", [448, 6])
def test_scale_exponent_matches_exact_rule(q):
    rng = np.random.default_rng(1)
    cases = list(rng.standard_normal(2000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 2000))
    for e in range(-60, 60):
        b = np.float32(q * 2.0 ** e)
        cases += [b, np.nextafter(b, np.float32(np.inf)), np.nextafter(b, np.float32(0))]
    for v in cases:
        a = abs(float(np.float32(v)))
        if a == 0:
            continue
        assert oracle.scale_exponent(a, float(q)) == exact_exponent(a, q), a


def test_scale_exponent_special_cases():
    assert oracle.scale_exponent(0.0, 448.0) == 0          # amax = 0 -> scale byte 127
    assert oracle.scale_exponent(448.0, 448.0) == 0
    assert oracle.scale_exponent(448.00003, 448.0) == 1
    assert oracle.scale_exponent(224.0, 448.0) == -1
    assert oracle.scale_exponent(6.0, 6.0) == 0
    assert oracle.scale_exponent(3.0000002, 6.0) == 0
    assert oracle.scale_exponent(1e-45, 448.0) == -127      # clamped at scale byte 0


def test_round_e4m3_matches_torch_rne():
    rng = np.random.default_rng(2)
    vals = [rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 0.01,
            rng.standard_normal(20000) * 2.0 ** -8]
    # every midpoint between adjacent non-negative E4M3 values (the ties)
    pos = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (pos[1:] + pos[:-1]) / 2
    vals += [mids, -mids]
    v = np.concatenate(vals).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.round_e4m3(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(ref, mine)


def test_round_e2m1_matches_brute_force_nearest():
    def nearest(v):
        best = None
        for code in range(16):
            val = (-1 if code & 8 else 1) * OCP_E2M1[code & 7]
            if (code & 8) != (8 if np.signbit(v) else 0):
                continue
            d = abs(v - val)
            key = (d, code & 1)  # ties: even mantissa bit
            if best is None or key < best[0]:
                best = (key, code)
        return best[1]
    grid = [i / 64.0 for i in range(-6 * 64, 6 * 64 + 1)] + [-0.0]
    for v in grid:
        assert oracle.round_e2m1(v) == nearest(v), v


def test_quantize_e4m3_round_trip_and_rule():
    rng = np.random.default_rng(3)
    pos = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    rows = []
    for e in (-20, -3, 0, 5):
        codes = rng.integers(0, 127, 32)
        codes[rng.integers(32)] = 126  # 448: forces exponent e
        sign = np.where(rng.random(32) < 0.5, -1.0, 1.0)
        rows.append(sign * pos[codes] * 2.0 ** e)
    src = np.array(rows, dtype=np.float32)
    q, sf = oracle.quantize_e4m3(src)
    assert list(sf[:, 0]) == [127 - 20, 127 - 3, 127, 127 + 5]
    back = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy() * 2.0 ** (sf.astype(np.float64) - 127)
    assert np.array_equal(back, src.astype(np.float64))


def test_quantize_e4m3_random_matches_rule():
    rng = np.random.default_rng(4)
    src = (rng.standard_normal((33, 128)) * 0.5).astype(np.float32)
    src[0, :32] = 0.0
    q, sf = oracle.quantize_e4m3(src)
    assert np.all(q[0, :32] == 0) and sf[0, 0] == 127
    g = src.reshape(33, 4, 32)
    for r in range(33):
        for j in range(4):
            amax = float(np.abs(g[r, j]).max())
            if amax > 0:
                assert sf[r, j] == exact_exponent(amax, 448) + 127
    scale = 2.0 ** (sf.astype(np.float64) - 127)
    ref = torch.from_numpy((g / scale[:, :, None]).astype(np.float32).reshape(33, 128)).to(torch.float8_e4m3fn)
    assert np.array_equal(ref.view(torch.uint8).numpy(), q)


def test_quantize_e2m1_packing_and_rule():
    rng = np.random.default_rng(5)
    src = (rng.standard_normal((9, 64)) * 0.04).astype(np.float32)
    packed, sf = oracle.quantize_e2m1(src)
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.empty((9, 64), np.uint8)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    vals = np.array([(-1 if c & 8 else 1) * OCP_E2M1[c & 7] for c in range(16)])
    g = src.reshape(9, 2, 32)
    for r in range(9):
        for j in range(2):
            amax = float(np.abs(g[r, j]).max())
            e = exact_exponent(amax, 6)
            assert sf[r, j] == e + 127
            for i in range(32):
                v = float(g[r, j, i]) / 2.0 ** e
                d = np.abs(vals - v)
                # nearest value; on a tie the even code
                best = min(range(16), key=lambda c: (d[c], c & 1, (c & 8) != (8 if np.signbit(v) else 0)))
                assert vals[codes[r, j * 32 + i]] == vals[best]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(6)
    v = np.concatenate([rng.standard_normal(5000).astype(np.float32),
                        # exact ties: bf16 value + half an ulp
                        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x18000).view(np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(oracle.f32_to_bf16(v), ref)
