"""Pins for the oracle's format decoders (not the oracle's own formulas):
E4M3 against torch's float8_e4m3fn conversion, E2M1 against the OCP
Microscaling v1.0 element table, UE8M0 against ldexp and torch's float8_e8m0fnu.
"""
import math

import numpy as np
import pytest
import torch

import oracle

# OCP Microscaling Formats v1.0, FP4 E2M1 element encodings (sign, then the
# 3-bit magnitude code 000..111): 0, 0.5, 1, 1.5, 2, 3, 4, 6.
OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_all_256_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])
    assert max(mine[~nan]) == 448.0 and min(abs(mine[(mine != 0) & ~nan])) == 2.0 ** -9


def test_e2m1_all_16_codes_match_ocp_table():
    for c in range(16):
        v = oracle.e2m1_value(c)
        mag = OCP_E2M1[c & 7]
        assert v == (-mag if c & 8 else mag)
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)


def test_ue8m0_all_codes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for b in range(255):
        assert oracle.ue8m0_value(b) == math.ldexp(1.0, b - 127) == ref[b]
    assert math.isnan(oracle.ue8m0_value(255)) and math.isnan(ref[255])
