"""Pins for the oracle on general NVFP4 sources: e4m3 block scales and an fp32
scale_2 that are not powers of two (not the output of the MXFP4 conversion).

Source: "DeepSeek-v4-Flash-REAP-K180-NVFP4", section "NVFP4: lossless
MXFP4->NVFP4 conversion": NVFP4 = e2m1 nibbles, one e4m3 scale per 16
elements and one fp32 scale_2 per expert; a weight is e2m1 * e4m3 * scale_2.

Checked against: a hand-worked block (tests/golden/nvfp4_general_block.txt),
the library decoders of ml_dtypes with numpy products over every non-NaN e4m3
code, and invariants of the product form (a uniform block scale moved into
scale_2, power-of-two covariance of the down projection's scale_2).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from block_quantized_expert_mxfp4_b200 import synth
from conftest import golden
from helpers import NV, oracle_moe
from ref_decode import E4M3, bf16_to_f64, dequant_nv

NAN_FREE = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)


def _read_golden():
    d = {}
    for line in open(golden("nvfp4_general_block.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            key, *vals = line.split()
            d[key] = vals
    return d


def _one_row(q, e4, s2):
    return oracle.Weight(oracle.NVFP4, q.reshape(1, 1, -1), e4.reshape(1, 1, -1),
                         np.asarray([s2], np.float32))


def test_worked_general_block():
    g = _read_golden()
    q = np.array([int(b, 16) for b in g["bytes"]], np.uint8)
    e4 = np.array([int(b, 16) for b in g["e4m3"]], np.uint8)
    dq = oracle.dequant(_one_row(q, e4, float(g["scale_2"][0])), 0)[0]
    want = np.array([float(v) for v in g["dequant"]])
    assert np.array_equal(dq, want)
    assert all(math.copysign(1, a) == math.copysign(1, b) for a, b in zip(dq, want))
    j = np.arange(32)
    half = (j % 16 < 8).astype(np.float64)
    assert float(dq @ half) == float(g["dot_half_ones"][0])
    assert float(dq @ (2 * half - 1)) == float(g["dot_plus_minus"][0])
    assert float(dq @ np.ones(32)) == float(g["dot_all_ones"][0])


def test_worked_block_scale_2_not_rounded_to_fp32():
    g = _read_golden()
    q = np.array([int(b, 16) for b in g["bytes"]], np.uint8)
    e4 = np.array([int(b, 16) for b in g["e4m3"]], np.uint8)
    s2 = np.array([int(g["tenth_scale_2_bits"][0], 16)], np.uint32).view(np.float32)[0]
    dq = oracle.dequant(_one_row(q, e4, s2), 0)[0]
    want = float(g["tenth_element_7"][0])
    assert dq[7] == want
    assert float(np.float32(want)) != want  # the exact product is not an fp32 value


def test_dequant_matches_library_decoders_every_code():
    """Every non-NaN e4m3 code (zero, subnormals, both signs, 448) as a block
    scale, with non-power-of-two scale_2 values: bit-identical float64."""
    rng = np.random.default_rng(20)
    E, N, K = 3, 16, 512
    q = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    e4 = NAN_FREE[rng.integers(0, NAN_FREE.size, (E, N, K // 16))]
    e4.reshape(-1)[:NAN_FREE.size] = NAN_FREE       # each code at least once
    s2 = np.array([0.1, 3.0e-5, 7.77], np.float32)  # none a power of two
    want = dequant_nv(q, e4, s2)
    for e in range(E):
        got = oracle.dequant(oracle.Weight(oracle.NVFP4, q, e4, s2), e)
        assert np.array_equal(got.view(np.uint64), want[e].view(np.uint64))


def test_expert_ffn_matches_library_formulation():
    rng = np.random.default_rng(21)
    E, H, I = 2, 256, 128
    mats = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        q = rng.integers(0, 256, (E, rows, cols // 2), dtype=np.uint8)
        e4 = rng.integers(0x30, 0x7F, (E, rows, cols // 16)).astype(np.uint8)
        s2 = (rng.uniform(0.5, 1.0, E) * 2.0 ** -6).astype(np.float32)
        mats.append((q, e4, s2))
    L = oracle.Layer(*[oracle.Weight(oracle.NVFP4, *m) for m in mats])
    x = synth.activations(4, 2, H)
    for t in range(2):
        x64 = bf16_to_f64(x[t])
        for e in range(E):
            Wg, Wu, Wd = (dequant_nv(q[e:e + 1], e4[e:e + 1], s2[e:e + 1])[0] for q, e4, s2 in mats)
            g = Wg @ x64
            u = Wu @ x64
            d = Wd @ (g * expit(g) * u)
            got = oracle.expert_ffn(L, e, x[t])[3]
            np.testing.assert_allclose(got, d, rtol=1e-12, atol=1e-12 * np.abs(d).max())


@pytest.mark.parametrize("code", [0x3B, 0x55, 0x7E, 0x03])
def test_uniform_block_scale_moves_into_scale_2(code):
    """All block codes equal to `code` (value v) with scale_2 = s is the same
    matrix as all block codes 0x38 (= 1) with scale_2 = v * s (exact in fp32:
    s has 16 significant bits, v at most 4)."""
    rng = np.random.default_rng(22)
    E, N, K = 2, 8, 256
    q = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    s = np.array([0.7001953125, 1.2998046875 * 2.0 ** -20], np.float64)  # 16-bit significands
    v = E4M3[code]
    moved = (s * v).astype(np.float32)
    assert np.array_equal(moved.astype(np.float64), s * v)
    a = oracle.Weight(oracle.NVFP4, q, np.full((E, N, K // 16), code, np.uint8), s.astype(np.float32))
    b = oracle.Weight(oracle.NVFP4, q, np.full((E, N, K // 16), 0x38, np.uint8), moved)
    for e in range(E):
        assert np.array_equal(oracle.dequant(a, e), oracle.dequant(b, e))


def test_down_scale_2_covariance():
    """Multiplying the down projection's scale_2 by 2^j multiplies y by 2^j
    exactly (power-of-two scaling commutes with every rounding)."""
    rng = np.random.default_rng(23)
    E, H, I = 3, 128, 64
    mats = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        q = rng.integers(0, 256, (E, rows, cols // 2), dtype=np.uint8)
        e4 = rng.integers(0x40, 0x7F, (E, rows, cols // 16)).astype(np.uint8)
        s2 = rng.uniform(1e-4, 2e-4, E).astype(np.float32)
        mats.append((q, e4, s2))
    x = synth.activations(5, 2, H)
    ids = np.array([[0, 2], [1, 0]], np.int32)
    w = np.array([[0.7, 0.3], [0.25, 0.75]])
    y0 = oracle.moe_forward(oracle.Layer(*[oracle.Weight(oracle.NVFP4, *m) for m in mats]), x, ids, w)
    for j in (-7, 5):
        m2 = mats[:2] + [(mats[2][0], mats[2][1], (mats[2][2] * np.float32(2.0 ** j)))]
        y1 = oracle.moe_forward(oracle.Layer(*[oracle.Weight(oracle.NVFP4, *m) for m in m2]), x, ids, w)
        assert np.array_equal(y1, y0 * 2.0 ** j)


def test_nan_block_scale_is_an_error():
    q = np.zeros((1, 1, 16), np.uint8)
    for bad in (0x7F, 0xFF):
        e4 = np.full((1, 1, 2), 0x38, np.uint8)
        e4[0, 0, 1] = bad
        with pytest.raises(oracle.OracleError):
            oracle.dequant(oracle.Weight(oracle.NVFP4, q, e4, np.ones(1, np.float32)), 0)


# ------------------------------------------------ the seeded general source --

def test_generator_codes_and_scale_2():
    q, e4, s2 = synth.nv_expert_bytes(0, 0, synth.TID.GATE, 64, 512, None, 4)
    assert e4.shape == (4, 64, 32) and q.shape == (4, 64, 256)
    c = e4.numpy()
    assert c.min() == synth.NV_CODE_LO and c.max() == synth.NV_CODE_HI
    assert len(np.unique(c)) == synth.NV_CODE_HI - synth.NV_CODE_LO + 1
    v = s2.numpy().astype(np.float64)
    assert np.all((v >= 2.0 ** -13) & (v < 2.0 ** -12)) and len(np.unique(v)) == 4
    assert not np.any(np.log2(v) == np.round(np.log2(v)))  # not powers of two
    # the nibbles are the MXFP4 stream's; a slice equals the full tensor's
    qm, _ = synth.mx_expert_bytes(0, 0, synth.TID.GATE, 64, 512, 118, 127, None, 4)
    assert torch.equal(q, qm)
    q2, e42, s22 = synth.nv_expert_bytes(0, 0, synth.TID.GATE, 64, 512, [3, 1], 4)
    assert torch.equal(q2[0], q[3]) and torch.equal(e42[1], e4[1]) and s22[0] == s2[3]
    with pytest.raises(ValueError):
        synth.nv_expert_bytes(0, 0, 0, 8, 64, None, 1, code_lo=0, code_hi=0x7F)


def test_tiny_general_layer_through_the_test_helper():
    """The host side of the GPU parity tests for general NVFP4: the helper's
    sub-layer gives the library formulation's y."""
    wl = synth.WORKLOADS["tiny"]
    fmts, codes = (NV, NV, NV), (0x00, 0x7E)
    x = synth.activations(3, wl.T, wl.H)
    ids, w = oracle.route_topk(synth.router_logits(3, wl.T, wl.E), wl.k)
    y = oracle_moe(wl, 3, 0, x, ids, w, fmts, codes)
    shapes = ((wl.I, wl.H), (wl.I, wl.H), (wl.H, wl.I))
    mats = [synth.nv_expert_bytes(3, 0, p, r, c, None, wl.E, "cpu", *codes)
            for p, (r, c) in enumerate(shapes)]
    dq = [dequant_nv(q.numpy(), e4.numpy(), s2.numpy()) for q, e4, s2 in mats]
    x64 = bf16_to_f64(x)
    for t in range(wl.T):
        want = np.zeros(wl.H)
        for s in range(wl.k):
            e = ids[t, s]
            g = dq[0][e] @ x64[t]
            u = dq[1][e] @ x64[t]
            want += w[t, s] * (dq[2][e] @ (g * expit(g) * u))
        np.testing.assert_allclose(y[t], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
