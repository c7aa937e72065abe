"""Pins from the hand-worked block, the bits-per-weight figures and block geometry."""
import math

import numpy as np
import torch

import oracle
from conftest import golden


def _read_golden():
    d = {}
    for line in open(golden("mxfp4_worked_block.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        d[key] = vals
    return d


def _one_row_layer(q, s, fmt=oracle.MXFP4, s2=None):
    w = oracle.Weight(fmt, q.reshape(1, 1, -1), s.reshape(1, 1, -1), s2)
    return w


def test_worked_block_dequant_and_dots():
    g = _read_golden()
    q = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)
    s = np.array([int(g["scale"][0])], dtype=np.uint8)
    w = _one_row_layer(q, s)
    dq = oracle.dequant(w, 0)[0]
    want = np.array([float(v) for v in g["dequant"]], dtype=np.float32)
    assert np.array_equal(dq, want)
    assert all(math.copysign(1, a) == math.copysign(1, b) for a, b in zip(dq, want))
    j = np.arange(32)
    half = (j % 16 < 8).astype(np.float64)
    assert float(dq.astype(np.float64) @ half) == float(g["dot_half_ones"][0])
    assert float(dq.astype(np.float64) @ (2 * half - 1)) == float(g["dot_plus_minus"][0])
    assert float(dq.astype(np.float64) @ np.ones(32)) == float(g["dot_all_ones"][0])


def test_worked_block_nv_view():
    g = _read_golden()
    q = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)
    s = np.array([int(g["scale"][0])], dtype=np.uint8).reshape(1, 1, 1)
    e4, s2, bad = oracle.convert_mx_to_nv(s)
    assert bad == 0
    assert float(s2[0]) == float(g["nv_scale_2"][0])
    assert [f"{c:02X}" for c in e4.reshape(-1)] == g["nv_e4m3"]
    dq_mx = oracle.dequant(_one_row_layer(q, s.reshape(-1)), 0)
    dq_nv = oracle.dequant(_one_row_layer(q, e4.reshape(-1), oracle.NVFP4, s2), 0)
    assert np.array_equal(dq_mx.view(np.uint64), dq_nv.view(np.uint64))


def test_worked_block_ffn_dot_through_expert_path():
    """The same block as a 1-row gate of a one-hot-free expert: g = dot(x, dq)."""
    g = _read_golden()
    q = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)
    # a 32x32 layer whose gate row 0 is the worked block, everything else zero
    H = I = 32
    gq = np.zeros((1, I, H // 2), np.uint8)
    gq[0, 0] = q
    sc = np.full((1, I, 1), 126, np.uint8)
    zq = np.zeros((1, I, H // 2), np.uint8)
    dq_ = np.zeros((1, H, I // 2), np.uint8)
    L = oracle.Layer(oracle.Weight(oracle.MXFP4, gq, sc), oracle.Weight(oracle.MXFP4, zq, sc),
                     oracle.Weight(oracle.MXFP4, dq_, np.full((1, H, 1), 126, np.uint8)))
    j = np.arange(32)
    x = torch.tensor((2 * (j % 16 < 8) - 1).astype(np.float32)).to(torch.bfloat16)
    gg, _, _, _ = oracle.expert_ffn(L, 0, x)
    assert gg[0] == 36.0 and np.all(gg[1:] == 0.0)


def test_bits_per_weight_pins_block_sizes():
    """4.25 bpw (MXFP4) and 4.50 bpw (NVFP4, per-expert fp32 excluded) fix the
    block lengths 32 and 16 with one 8-bit scale each: changing one scale code
    changes exactly that many consecutive dequantized elements."""
    K = 128
    rng = np.random.default_rng(0)
    q = rng.integers(0, 256, (1, 1, K // 2), dtype=np.uint8)
    q |= 0x22  # no zero magnitudes, so every element sees its scale
    for fmt, blk, base, alt in ((oracle.MXFP4, 32, 120, 121), (oracle.NVFP4, 16, 0x38, 0x40)):
        s = np.full((1, 1, K // blk), base, np.uint8)
        s2 = np.ones(1, np.float32) if fmt == oracle.NVFP4 else None
        ref = oracle.dequant(oracle.Weight(fmt, q, s, s2), 0)[0]
        for b in range(K // blk):
            s_b = s.copy()
            s_b[0, 0, b] = alt
            dq = oracle.dequant(oracle.Weight(fmt, q, s_b, s2), 0)[0]
            changed = np.nonzero(dq != ref)[0]
            assert list(changed) == list(range(b * blk, (b + 1) * blk))
        bpw = (q.size * 8 + s.size * 8) / K
        assert bpw == {32: 4.25, 16: 4.5}[blk]


def test_gate_up_are_two_thirds_of_expert_bytes():
    """'gate+up ~2/3 of expert bytes' (REAP-K180 page): three equal matrices."""
    H, I = 4096, 2048
    per = lambda rows, cols: rows * cols // 2 + rows * cols // 32
    gate, up, down = per(I, H), per(I, H), per(H, I)
    assert gate == up == down
    assert (gate + up) / (gate + up + down) == 2 / 3
    assert gate + up + down == 13_369_344
