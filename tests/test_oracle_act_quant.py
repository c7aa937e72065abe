"""Pins for the oracle's activation-quantized modes (MXFP4 or E4M3
activations with one e8m0 scale per 32, the OCP Microscaling scale rule).

Source for the mode: "DeepSeekv4 Flash for 1x Spark [REAP25]", v0.2.3 update
(fp4 weights x dynamic E4M3 activations on the block-scaled f8f6f4 tensor
cores).  The scale rule is the reading adopted where the pages give none.

Checked against: hand-worked blocks (tests/golden/act_quant_blocks.txt), the
ml_dtypes casts, a brute-force nearest-code search over each format's code
table, the rule's own invariants (where the block maximum lands, power-of-two
covariance, idempotence), and a second formulation of the FFN built from
ml_dtypes casts and numpy products.
"""
import ml_dtypes
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from block_quantized_expert_mxfp4_b200 import synth
from conftest import golden
from ref_decode import E2M1, E4M3, bf16_to_f64, dequant_mx

MODES = {"mxfp4": oracle.ACT_MXFP4, "e4m3": oracle.ACT_E4M3}
GRID = {oracle.ACT_MXFP4: (E2M1, np.arange(16)), oracle.ACT_E4M3: (E4M3, np.array(
    [c for c in range(256) if c & 0x7F != 0x7F]))}
TOP = {oracle.ACT_MXFP4: (4.0, 6.0), oracle.ACT_E4M3: (256.0, 448.0)}


def _fixture():
    for line in open(golden("act_quant_blocks.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, vals, want = (p.split() for p in line.split("|"))
        name, mode, code = head
        v = np.zeros(32)
        v[:len(vals)] = [float(t) for t in vals]
        w = np.zeros(32)
        w[:len(want)] = [float(t) for t in want]
        yield name, MODES[mode], int(code), v, w


def test_hand_worked_blocks():
    n = 0
    for name, aq, code, v, want in _fixture():
        _, scales, out = oracle.act_quant(v, aq)
        assert scales[0] == code, name
        assert np.array_equal(out, want), (name, out[:8])
        n += 1
    assert n == 6


def test_e2m1_encode_matches_library_cast():
    vals = np.concatenate([np.arange(-160, 161) / 16.0,                  # every midpoint of the grid
                           np.random.default_rng(0).uniform(-9, 9, 5000),
                           [0.0, -0.0, 1e-300, -1e-300, 6.0, 6.0001, 1e30, -1e30]])
    want = vals.astype(ml_dtypes.float4_e2m1fn)  # RNE, saturating
    for v, w in zip(vals, want):
        c = oracle.e2m1_encode(v)
        assert E2M1[c] == float(w) and np.signbit(E2M1[c]) == np.signbit(float(w)), v


def _nearest_even(q, table, codes):
    """Brute force: the code whose value is nearest q; on a tie the code with
    mantissa bit 0 (even); values beyond the largest saturate."""
    vals = table[codes]
    d = np.abs(vals - q)
    best = codes[d == d.min()]
    if best.size > 1:
        best = best[best % 2 == 0]
    return table[best[0]]


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
def test_elements_are_the_nearest_code_brute_force(aq):
    table, codes = GRID[aq]
    rng = np.random.default_rng(1)
    for trial in range(60):
        v = rng.standard_normal(32) * 2.0 ** rng.integers(-5, 6, 32) * 2.0 ** rng.integers(-30, 30)
        _, scales, out = oracle.act_quant(v, aq)
        s = 2.0 ** (int(scales[0]) - 127)
        top = TOP[aq][1]
        for x, got in zip(v, out):
            q = x / s
            want = np.sign(q) * top if abs(q) >= top else _nearest_even(q, table, codes)
            assert got / s == want or (got == 0 and want == 0), (trial, x, got, want)


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
def test_block_maximum_lands_in_the_top_binade(aq):
    """The scale puts each block's largest magnitude in [4, 8) (e2m1) or
    [256, 512) (e4m3) before the cast, so after it in [4, 6] or [256, 448]:
    a scale off by one binade either way breaks this."""
    lo, hi = TOP[aq]
    rng = np.random.default_rng(2)
    v = rng.standard_normal(32 * 400) * 2.0 ** rng.integers(-40, 40, 32 * 400).repeat(1)
    _, scales, out = oracle.act_quant(v, aq)
    q = np.abs(out.reshape(-1, 32)) / 2.0 ** (scales.astype(np.int64) - 127)[:, None]
    assert np.all((q.max(1) >= lo) & (q.max(1) <= hi))
    pre = np.abs(v.reshape(-1, 32)).max(1) / 2.0 ** (scales.astype(np.int64) - 127)
    assert np.all((pre >= lo) & (pre < 2 * lo))


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
def test_power_of_two_covariance_and_idempotence(aq):
    rng = np.random.default_rng(3)
    v = rng.standard_normal(32 * 50)
    c0, s0, o0 = oracle.act_quant(v, aq)
    for j in (-20, 7):
        c1, s1, o1 = oracle.act_quant(v * 2.0 ** j, aq)
        assert np.array_equal(c1, c0) and np.array_equal(s1.astype(int), s0.astype(int) + j)
        assert np.array_equal(o1, o0 * 2.0 ** j)
    c2, s2, o2 = oracle.act_quant(o0, aq)
    assert np.array_equal(o2, o0) and np.array_equal(s2, s0)


def test_invalid_inputs():
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(np.ones(33), oracle.ACT_MXFP4)
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(np.ones(32), 7)
    v = np.ones(32)
    v[3] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(v, oracle.ACT_E4M3)


# -------------------------------------------------------------- the FFN --

def _lib_quant(v, aq):
    """Second formulation: X from np.frexp, elements by the ml_dtypes casts
    (e4m3 saturated by clipping first: the library cast overflows to NaN)."""
    b = v.reshape(-1, 32)
    amax = np.abs(b).max(1)
    _, ex = np.frexp(amax)
    X = np.where(amax > 0, np.clip(ex - 1 - (2 if aq == oracle.ACT_MXFP4 else 8), -127, 127), -127)
    q = b / 2.0 ** X[:, None]
    if aq == oracle.ACT_MXFP4:
        e = q.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    else:
        e = np.clip(q, -448, 448).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return (e * 2.0 ** X[:, None]).reshape(v.shape)


def _layer(E, H, I, seed):
    rng = np.random.default_rng(seed)
    ws = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        ws.append((rng.integers(0, 256, (E, rows, cols // 2), dtype=np.uint8),
                   rng.integers(118, 128, (E, rows, cols // 32), dtype=np.uint8)))
    return ws, oracle.Layer(*[oracle.Weight(oracle.MXFP4, q, s) for q, s in ws])


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
def test_ffn_matches_library_formulation(aq):
    E, H, I = 3, 256, 128
    ws, L = _layer(E, H, I, 4)
    x = synth.activations(6, 3, H)
    ids = np.array([[0, 2], [1, 0], [2, 1]], np.int32)
    w = np.array([[0.7, 0.3], [0.5, 0.5], [0.1, 0.9]])
    y = oracle.moe_forward(L, x, ids, w, aq)
    x64 = bf16_to_f64(x)
    for t in range(3):
        xq = _lib_quant(x64[t], aq)
        want = np.zeros(H)
        for s in range(2):
            e = ids[t, s]
            Wg, Wu, Wd = (dequant_mx(q[e], sc[e]) for q, sc in ws)
            g, u = Wg @ xq, Wu @ xq
            h = (g * expit(g) * u).astype(np.float32).astype(np.float64)
            hq = _lib_quant(h, aq)
            want += w[t, s] * (Wd @ hq)
            gg, uu, hh, dd = oracle.expert_ffn(L, e, x[t], aq)
            np.testing.assert_allclose(gg, g, rtol=1e-12, atol=1e-12 * np.abs(g).max())
            # the fp64 sums agree far below fp32 resolution, so the fp32 h and
            # its codes agree exactly on these seeded inputs
            assert np.array_equal(hh, hq)
        np.testing.assert_allclose(y[t], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_inputs_on_the_grid_pass_gate_up_unchanged():
    """x whose 32-blocks are already MXFP4 values with block maximum 4 or 6
    (times a power of two): quantization leaves x, so g and u, unchanged."""
    E, H, I = 1, 256, 64
    ws, L = _layer(E, H, I, 5)
    rng = np.random.default_rng(7)
    v = E2M1[rng.integers(0, 16, H)].reshape(-1, 32)
    v[:, 0] = rng.choice([4.0, 6.0, -6.0], v.shape[0])
    v = (v * 2.0 ** rng.integers(-8, 8, (v.shape[0], 1))).reshape(-1)
    x = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(bf16_to_f64(x), v)
    g0, u0, _, _ = oracle.expert_ffn(L, 0, x)
    g1, u1, _, _ = oracle.expert_ffn(L, 0, x, oracle.ACT_MXFP4)
    assert np.array_equal(g0, g1) and np.array_equal(u0, u1)


def test_aq_none_is_the_plain_path():
    E, H, I = 2, 128, 64
    _, L = _layer(E, H, I, 8)
    x = synth.activations(2, 2, H)
    ids = np.array([[0, 1], [1, 0]], np.int32)
    w = np.array([[0.5, 0.5], [0.25, 0.75]])
    assert np.array_equal(oracle.moe_forward(L, x, ids, w), oracle.moe_forward(L, x, ids, w, oracle.ACT_NONE))


def test_h_is_rounded_to_fp32_before_it_is_quantized():
    """A constructed expert whose h lies within fp32 rounding of an e2m1 tie.
    g = 40 and 64 (silu(g) = g exactly in fp64 for g >= 38), u = 1 + 2^-25
    and 1: h = 40 + 40 * 2^-25 and 64.  The block maximum 64 gives X = 4.
    fp32(h) = 40 exactly (half an fp32 ulp at 40 is 2^-19 > 40 * 2^-25), and
    40 / 16 = 2.5 is a tie between 2 and 3 that goes to the even code: 2, so
    hq = 32.  Without the fp32 rounding h / 16 lies above the tie and gives
    3 (48).  down row 0 picks hq at that index."""
    H = I = 64
    qg, qu, qd = (np.zeros((1, r, c // 2), np.uint8) for r, c in ((I, H), (I, H), (H, I)))
    sg, su, sd = (np.full((1, r, c // 32), 127, np.uint8) for r, c in ((I, H), (I, H), (H, I)))

    def put(q, s, row, col, code, scale):
        q[0, row, col // 2] |= code << (4 * (col % 2))
        s[0, row, col // 32] = scale

    put(qg, sg, 0, 0, 6, 131)   # g_0 = 4 * 2^4 = 64
    put(qu, su, 0, 0, 2, 127)   # u_0 = 1
    put(qg, sg, 1, 0, 6, 130)   # g_1 = 4 * 2^3 + 1 * 2^3 = 40
    put(qg, sg, 1, 32, 2, 130)
    put(qu, su, 1, 0, 2, 127)   # u_1 = 1 + 0.5 * 2^-24 = 1 + 2^-25
    put(qu, su, 1, 32, 1, 103)
    put(qd, sd, 0, 1, 2, 127)   # d_0 = hq_1
    L = oracle.Layer(oracle.Weight(oracle.MXFP4, qg, sg), oracle.Weight(oracle.MXFP4, qu, su),
                     oracle.Weight(oracle.MXFP4, qd, sd))
    x = torch.zeros(H, dtype=torch.bfloat16)
    x[0] = x[32] = 1.0
    g, u, h, d = oracle.expert_ffn(L, 0, x, oracle.ACT_MXFP4)
    assert g[0] == 64 and g[1] == 40 and u[1] == 1 + 2.0 ** -25
    assert h[0] == 64 and h[1] == 32 and d[0] == 32
    _, _, h_plain, _ = oracle.expert_ffn(L, 0, x)
    assert h_plain[1] == 40 + 40 * 2.0 ** -25
