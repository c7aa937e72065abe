"""Pins for the oracle's element codes, against library decoders and closed forms.

The pages name e2m1, e8m0/UE8M0 and E4M3 but print no bit tables; the
oracle's tables are pinned here to ml_dtypes' and torch's independent decoders
(OCP Microscaling v1.0 / E4M3FN definitions), over every code.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle


def test_e2m1_all_16_codes_match_library():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert v == lib[c] and math.copysign(1, v) == math.copysign(1, lib[c]), c


def test_e2m1_magnitudes_closed_form():
    mags = [oracle.e2m1_value(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert math.copysign(1, oracle.e2m1_value(8)) == -1.0  # code 8 is -0


def test_e8m0_all_256_codes_match_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    tl = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for c in range(255):
        assert oracle.e8m0_value(c) == lib[c] == tl[c] == math.ldexp(1.0, c - 127), c
    assert math.isnan(oracle.e8m0_value(255))


def test_e4m3_all_256_codes_match_two_libraries():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tl = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(v) and math.isnan(lib[c]) and math.isnan(tl[c])
        else:
            assert v == lib[c] == tl[c], c
            assert math.copysign(1, v) == math.copysign(1, lib[c])
    assert oracle.e4m3_value(0x7E) == 448.0
    # the 18 exact powers of two 2^-9 .. 2^8
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x02) == 2.0 ** -8
    assert oracle.e4m3_value(0x04) == 2.0 ** -7
    for d in range(-6, 9):
        assert oracle.e4m3_value((d + 7) << 3) == 2.0 ** d


def _lib_cast(v):
    """RNE cast by ml_dtypes (saturation is checked separately)."""
    return int(np.array([v], dtype=np.float64).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0])


def test_e4m3_encode_powers_of_two_match_library():
    for d in range(-14, 9):
        v = 2.0 ** d
        assert oracle.e4m3_encode(v) == _lib_cast(v), d
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 0x01


def test_e4m3_encode_random_in_range_match_library():
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.uniform(-448, 448, 4000),
                           rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 6, 4000)])
    for v in vals:
        assert oracle.e4m3_encode(float(v)) == _lib_cast(float(v)), v


def test_e4m3_encode_saturates_and_roundtrips():
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-1e9) == 0xFE
    assert oracle.e4m3_encode(470.0) == 0x7E
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c, c
