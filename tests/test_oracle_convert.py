"""Pins for the scale-only MXFP4 -> NVFP4 conversion.

Source: "DeepSeek-v4-Flash-REAP-K180-NVFP4", section "NVFP4: lossless
MXFP4->NVFP4 conversion": the e2m1 nibbles are kept, only the scales change,
and the result is lossless.  The anchor-at-max rule is the reading adopted for
the unstated choice of scale_2; these tests pin what any lossless rule must
satisfy (identical dequantized values) plus the rule's stated edge cases.
"""
import numpy as np
import pytest

import oracle
from conftest import golden
from ref_decode import E4M3, E8M0, dequant_mx, dequant_nv


def _rand(E, N, K, lo, hi, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    s = rng.integers(lo, hi + 1, (E, N, K // 32), dtype=np.uint8)
    return q, s


@pytest.mark.parametrize("lo,hi", [(118, 127), (121, 129), (0, 17), (237, 254), (100, 100)])
def test_lossless_when_span_le_17(lo, hi):
    q, s = _rand(3, 8, 128, lo, hi)
    e4, s2, bad = oracle.convert_mx_to_nv(s)
    assert bad == 0
    a = dequant_mx(q, s)
    b = dequant_nv(q, e4, s2)
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))
    # and through the oracle's own dequant
    for e in range(3):
        da = oracle.dequant(oracle.Weight(oracle.MXFP4, q, s), e)
        db = oracle.dequant(oracle.Weight(oracle.NVFP4, q, e4, s2), e)
        assert np.array_equal(da.view(np.uint64), db.view(np.uint64))


def test_scale2_is_power_of_two_anchor_at_max():
    q, s = _rand(4, 4, 64, 118, 127, seed=3)
    e4, s2, _ = oracle.convert_mx_to_nv(s)
    for e in range(4):
        cmax = int(s[e].max())
        assert s2[e] == np.float32(2.0 ** (cmax - 127 - 8))
        # every e4m3 code is a power of two 2^(c - cmax + 8), equal in both halves
        assert np.array_equal(e4[e, :, 0::2], e4[e, :, 1::2])
        assert np.array_equal(E4M3[e4[e, :, 0::2]], 2.0 ** (s[e].astype(np.int64) - cmax + 8))


def test_span_17_exact_span_18_counts_inexact_blocks():
    s = np.full((1, 2, 4), 150, np.uint8)
    s[0, 0, 1] = 150 - 17
    e4, s2, bad = oracle.convert_mx_to_nv(s)
    assert bad == 0 and E4M3[e4[0, 0, 2]] == 2.0 ** -9
    s[0, 1, 3] = 150 - 18          # 2^-10: tie between 0 and 2^-9 -> 0
    s[0, 1, 2] = 150 - 30          # far below: 0
    e4, s2, bad = oracle.convert_mx_to_nv(s)
    assert bad == 2
    assert e4[0, 1, 6] == 0 and e4[0, 1, 7] == 0 and e4[0, 1, 4] == 0


def test_all_equal_codes_and_extremes():
    for c in (0, 1, 127, 254):
        s = np.full((2, 3, 2), c, np.uint8)
        e4, s2, bad = oracle.convert_mx_to_nv(s)
        assert bad == 0 and np.all(e4 == 0x78)
        assert s2[0] == np.float32(2.0 ** (c - 135)) and s2[0] != 0.0  # 2^-135 subnormal, exact
        assert float(s2[0]) * 256.0 == E8M0[c]


def test_nan_scale_rejected():
    s = np.full((1, 2, 2), 120, np.uint8)
    s[0, 1, 1] = 255
    with pytest.raises(oracle.OracleError) as ei:
        oracle.convert_mx_to_nv(s)
    assert ei.value.code == oracle.QKO_ERR_NAN_SCALE


def test_each_expert_independent():
    q, s = _rand(3, 4, 64, 118, 127, seed=5)
    e4, s2, _ = oracle.convert_mx_to_nv(s)
    for e in range(3):
        e4e, s2e, _ = oracle.convert_mx_to_nv(s[e:e + 1])
        assert np.array_equal(e4e[0], e4[e]) and s2e[0] == s2[e]


# --------------------------------------------------- NVFP4 -> MXFP4 (reverse) --

def test_reverse_hand_worked_cases():
    n = 0
    for line in open(golden("nv_to_mx_cases.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        s0, s1, s2, code, inexact = int(line[0], 16), int(line[1], 16), float(line[2]), int(line[3]), int(line[4])
        out, bad = oracle.convert_nv_to_mx(np.array([[[s0, s1]]], np.uint8), np.array([s2], np.float32))
        assert (int(out[0, 0, 0]), bad) == (code, inexact), line
        n += 1
    assert n == 11


@pytest.mark.parametrize("lo,hi", [(118, 127), (121, 129), (0, 17), (237, 254), (100, 100)])
def test_reverse_of_a_lossless_conversion_is_the_identity(lo, hi):
    q, s = _rand(3, 8, 128, lo, hi, seed=5)
    e4, s2, bad = oracle.convert_mx_to_nv(s)
    assert bad == 0
    back, bad2 = oracle.convert_nv_to_mx(e4, s2)
    assert bad2 == 0 and np.array_equal(back, s)


def test_reverse_general_sources_nearest_code_brute_force():
    """General NVFP4 (every non-NaN e4m3 code, scale_2 not a power of two):
    exact blocks dequantize identically in both formats; every inexact block
    takes the code nearest in log2 to its larger half scale, found here by
    trying all 255 codes."""
    rng = np.random.default_rng(6)
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    E, N, K = 3, 16, 256
    e4 = codes[rng.integers(0, codes.size, (E, N, K // 16))]
    e4[0, :4] = 0x38                      # some exact blocks: equal halves, scale_2 a power of two
    s2 = np.array([2.0 ** -5, 0.3, 7.0], np.float32)
    out, bad = oracle.convert_nv_to_mx(e4, s2)
    a = E4M3[e4[..., 0::2]] * s2[:, None, None].astype(np.float64)
    b = E4M3[e4[..., 1::2]] * s2[:, None, None].astype(np.float64)
    cand = 2.0 ** (np.arange(255) - 127.0)
    n_inexact = 0
    q = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    for idx in np.ndindex(a.shape):
        exact = a[idx] == b[idx] and a[idx] > 0 and a[idx] in cand
        if exact:
            assert cand[out[idx]] == a[idx]
            continue
        n_inexact += 1
        v = max(abs(a[idx]), abs(b[idx]))
        want = 0 if v == 0 else int(np.argmin(np.abs(np.log2(cand) - np.log2(v))))
        assert out[idx] == want, (idx, v, out[idx], want)
    assert bad == n_inexact and 0 < bad < a.size
    # exact blocks: the same dequantized values in both formats
    dm, dn = dequant_mx(q, out), dequant_nv(q, e4, s2)
    ex = np.repeat((a == b) & np.isin(a, cand), 32, axis=-1)
    assert np.array_equal(dm[ex], dn[ex])


def test_reverse_nan_code_is_an_error():
    for bad in (0x7F, 0xFF):
        with pytest.raises(oracle.OracleError):
            oracle.convert_nv_to_mx(np.array([[[0x38, bad]]], np.uint8), np.ones(1, np.float32))
