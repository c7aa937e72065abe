"""The activation terms of the block-scaled paths, checked on the CPU against
the exact arithmetic they claim (no GPU, no code shared with the kernels).

A block of 32 values v is written as a sum of e4m3 terms with one ue8m0 scale
per term and block: t_i = RN_e4m3(r_i / 2^(c_i - 127)), r_0 = v,
r_{i+1} = r_i - t_i 2^(c_i - 127), c_i = (biased exponent of max |r_i|) - 7.
Claims pinned here: two terms reproduce any bf16 block exactly, except values
below 2^-13 of the block's largest (absolute error there below 2^-20 of it);
three terms leave an fp32 value with relative error below 2^-12 (same
exception).
"""
import numpy as np


def _rn_e4m3(a):
    """Round float64 values to E4M3FN (bias 7, 3 mantissa bits, max 448,
    subnormals m/8 * 2^-6) with round-to-nearest-even; saturate at 448."""
    a = np.asarray(a, np.float64)
    out = np.zeros_like(a)
    nz = a != 0
    mag = np.abs(a[nz])
    e = np.floor(np.log2(mag))
    e = np.maximum(e, -6)                 # subnormal range shares the 2^-9 quantum
    q = np.exp2(e - 3)                    # quantum of the binade
    r = np.round(mag / q) * q             # numpy rounds half to even
    out[nz] = np.sign(a[nz]) * np.minimum(r, 448.0)
    return out


def _code(m):
    """ue8m0 code putting a positive fp32 maximum m into [128, 256)."""
    ef = (np.float32(m).view(np.uint32) >> 23) & 0xFF
    return int(min(max(int(ef) - 7, 0), 254))


def _split(v, terms):
    v = np.asarray(v, np.float32).astype(np.float64)
    r = v.copy()
    acc = np.zeros_like(v)
    for _ in range(terms):
        c = _code(np.abs(r).max())
        s = 2.0 ** (c - 127)
        t = _rn_e4m3(r / s)
        assert np.all(np.abs(t) <= 256.0)  # the scale choice keeps every term clear of saturation
        acc += t * s
        r = v - acc
    return v, acc


def _bf16(x):
    u = np.asarray(x, np.float32).view(np.uint32)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000  # round to nearest even
    return u.view(np.float32)


def test_two_terms_reproduce_bf16_blocks():
    rng = np.random.default_rng(0)
    for trial in range(3000):
        scale = 2.0 ** rng.integers(-40, 40)
        if trial % 3 == 0:
            x = rng.standard_normal(32) * scale
        elif trial % 3 == 1:
            x = rng.standard_normal(32) * 2.0 ** rng.integers(-6, 7, size=32) * scale  # wide in-block range
        else:
            x = rng.uniform(-1, 1, 32) * scale
        v, acc = _split(_bf16(x), 2)
        m = np.abs(v).max()
        big = np.abs(v) >= m * 2.0 ** -13
        assert np.array_equal(acc[big], v[big]), trial
        assert np.all(np.abs(acc - v) <= m * 2.0 ** -20), trial


def test_two_terms_edge_blocks():
    for x in (np.zeros(32), np.full(32, 448.0), np.full(32, -3.0e38),
              np.array([1.0] + [2.0 ** -126] * 31), np.array([2.0 ** -130] * 32)):
        v, acc = _split(_bf16(x), 2)
        m = np.abs(v).max()
        big = np.abs(v) >= m * 2.0 ** -13
        assert np.array_equal(acc[big], v[big])


def test_three_terms_bound_fp32_error():
    rng = np.random.default_rng(1)
    worst = 0.0
    for trial in range(3000):
        x = (rng.standard_normal(32) * 2.0 ** rng.integers(-3, 4, size=32)).astype(np.float32)
        x *= np.float32(2.0 ** rng.integers(-30, 30))
        v, acc = _split(x, 3)
        m = np.abs(v).max()
        big = np.abs(v) >= m * 2.0 ** -13
        rel = np.abs(acc[big] - v[big]) / np.abs(v[big])
        worst = max(worst, float(rel.max()))
        assert np.all(np.abs(acc[~big] - v[~big]) <= m * 2.0 ** -20), trial
    assert worst <= 2.0 ** -12, worst


def test_one_term_is_not_enough():
    """Sanity of the check itself: a single e4m3 term does not reproduce bf16."""
    rng = np.random.default_rng(2)
    v, acc = _split(_bf16(rng.standard_normal(32)), 1)
    assert not np.array_equal(acc, v)
