"""Pins for the oracle's routed-expert FFN, router and FP8 block linear.

Checked against: a second formulation built from library decoders and numpy /
scipy (decode the whole matrix, np.matmul, scipy.special.expit), exact
integer products, one-hot inputs, and invariants (power-of-two scale
covariance, expert relabelling, k=1 reduction, renormalised weights).
"""
import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

import oracle
from block_quantized_expert_mxfp4_b200 import synth
from ref_decode import bf16_to_f64, dequant_fp8, dequant_mx, dequant_nv


def _layer(E, H, I, lo, hi, seed=0):
    rng = np.random.default_rng(seed)
    ws = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        q = rng.integers(0, 256, (E, rows, cols // 2), dtype=np.uint8)
        s = rng.integers(lo, hi + 1, (E, rows, cols // 32), dtype=np.uint8)
        ws.append((q, s))
    return ws


def _oracle_layer(ws, fmt=oracle.MXFP4, s2s=(None, None, None)):
    return oracle.Layer(*[oracle.Weight(fmt, q, s, s2) for (q, s), s2 in zip(ws, s2s)])


def _ref_expert(ws, e, x64, nv=None):
    if nv is None:
        Wg, Wu, Wd = (dequant_mx(q[e], s[e]).astype(np.float64) for q, s in ws)
    else:
        Wg, Wu, Wd = (dequant_nv(q[e:e + 1], s4[e:e + 1], s2[e:e + 1])[0].astype(np.float64)
                      for (q, _), (s4, s2) in zip(ws, nv))
    g = Wg @ x64
    u = Wu @ x64
    h = g * expit(g) * u
    return g, u, h, Wd @ h


def test_expert_ffn_matches_library_formulation():
    E, H, I = 4, 256, 128
    ws = _layer(E, H, I, 121, 129)
    L = _oracle_layer(ws)
    x = synth.activations(0, 3, H)
    for t in range(3):
        x64 = bf16_to_f64(x[t])
        for e in range(E):
            got = oracle.expert_ffn(L, e, x[t])
            want = _ref_expert(ws, e, x64)
            for a, b in zip(got, want):
                np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12 * np.abs(b).max())


def test_one_hot_input_returns_a_column():
    E, H, I = 2, 64, 32
    ws = _layer(E, H, I, 118, 127, seed=1)
    L = _oracle_layer(ws)
    for k in (0, 5, 63):
        x = torch.zeros(H, dtype=torch.bfloat16)
        x[k] = 1.0
        g, u, _, _ = oracle.expert_ffn(L, 1, x)
        assert np.array_equal(g, dequant_mx(*ws[0])[1][:, k].astype(np.float64))
        assert np.array_equal(u, dequant_mx(*ws[1])[1][:, k].astype(np.float64))


def test_integer_weights_exact_product():
    """Scale code 127 (=1) and nibbles {0, 2} (values 0, 1): g and u are exact
    integer matrix products."""
    E, H, I = 1, 64, 32
    rng = np.random.default_rng(2)
    ws = []
    ints = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        bits = rng.integers(0, 2, (E, rows, cols)).astype(np.uint8) * 2
        q = (bits[..., 0::2] | (bits[..., 1::2] << 4)).astype(np.uint8)
        ws.append((q, np.full((E, rows, cols // 32), 127, np.uint8)))
        ints.append((bits // 2).astype(np.int64))
    L = _oracle_layer(ws)
    xi = rng.integers(-8, 9, H)
    x = torch.tensor(xi, dtype=torch.bfloat16)
    g, u, h, d = oracle.expert_ffn(L, 0, x)
    assert np.array_equal(g, (ints[0][0] @ xi).astype(np.float64))
    assert np.array_equal(u, (ints[1][0] @ xi).astype(np.float64))
    np.testing.assert_allclose(d, ints[2][0] @ h, rtol=1e-13)


def test_down_scale_shift_multiplies_output_by_power_of_two():
    E, H, I = 3, 128, 64
    ws = _layer(E, H, I, 118, 124, seed=4)
    x = synth.activations(1, 2, H)
    ids = np.array([[0, 2], [1, 0]], np.int32)
    w = np.array([[0.7, 0.3], [0.25, 0.75]])
    y0 = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    for j in (-5, 3):
        ws2 = [ws[0], ws[1], (ws[2][0], (ws[2][1].astype(np.int32) + j).astype(np.uint8))]
        y1 = oracle.moe_forward(_oracle_layer(ws2), x, ids, w)
        assert np.array_equal(y1, y0 * 2.0 ** j)


def test_expert_relabelling_invariance_and_k1_reduction():
    E, H, I = 5, 64, 32
    ws = _layer(E, H, I, 120, 127, seed=6)
    x = synth.activations(2, 3, H)
    ids = np.array([[4, 1, 0], [2, 3, 4], [0, 2, 1]], np.int32)
    w = np.array([[0.5, 0.3, 0.2], [0.1, 0.1, 0.8], [0.6, 0.2, 0.2]])
    y0 = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    perm = np.array([3, 0, 4, 1, 2])  # new slot of old expert e is perm[e]
    inv = np.argsort(perm)
    ws_p = [(q[inv], s[inv]) for q, s in ws]
    y1 = oracle.moe_forward(_oracle_layer(ws_p), x, perm[ids].astype(np.int32), w)
    assert np.array_equal(y0, y1)
    # k = 1 with weight 1 is the plain expert output
    L = _oracle_layer(ws)
    y = oracle.moe_forward(L, x[:1], np.array([[2]], np.int32), np.array([[1.0]]))
    assert np.array_equal(y[0], oracle.expert_ffn(L, 2, x[0])[3])


def test_moe_forward_matches_library_formulation_tiny_config():
    wl = synth.WORKLOADS["tiny"]
    ws = _layer(wl.E, wl.H, wl.I, wl.code_lo, wl.code_hi, seed=8)
    x = synth.activations(0, wl.T, wl.H)
    logits = synth.router_logits(0, wl.T, wl.E)
    ids, w = oracle.route_topk(logits, wl.k)
    y = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    x64 = bf16_to_f64(x)
    for t in range(wl.T):
        want = sum(w[t, s] * _ref_expert(ws, ids[t, s], x64[t])[3] for s in range(wl.k))
        np.testing.assert_allclose(y[t], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_nv_converted_layer_gives_identical_output():
    E, H, I = 4, 128, 64
    ws = _layer(E, H, I, 118, 127, seed=9)
    nv = [oracle.convert_mx_to_nv(s)[:2] for _, s in ws]
    x = synth.activations(3, 2, H)
    ids = np.array([[1, 3], [0, 1]], np.int32)
    w = np.array([[0.6, 0.4], [0.5, 0.5]])
    y_mx = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    L_nv = oracle.Layer(*[oracle.Weight(oracle.NVFP4, q, s4, s2)
                          for (q, _), (s4, s2) in zip(ws, nv)])
    y_nv = oracle.moe_forward(L_nv, x, ids, w)
    assert np.array_equal(y_mx, y_nv)
    g = _ref_expert(ws, 3, bf16_to_f64(x[0]), nv=nv)[3]
    np.testing.assert_allclose(oracle.expert_ffn(L_nv, 3, x[0])[3], g, rtol=1e-12,
                               atol=1e-12 * np.abs(g).max())


def test_nan_scale_is_an_error():
    E, H, I = 1, 64, 32
    ws = _layer(E, H, I, 120, 127)
    ws[1][1][0, 5, 1] = 255
    with pytest.raises(oracle.OracleError):
        oracle.moe_forward(_oracle_layer(ws), synth.activations(0, 1, H),
                           np.array([[0]], np.int32), np.array([[1.0]]))


# --------------------------------------------------------------- router --

def _ref_route(logits, k):
    p = softmax(logits.astype(np.float64), axis=1)
    ids = np.argsort(-p, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(p, ids, 1)
    return ids, sel / sel.sum(1, keepdims=True)


@pytest.mark.parametrize("T,E,k", [(4, 8, 2), (16, 256, 6), (8, 180, 6)])
def test_route_matches_library(T, E, k):
    lg = synth.router_logits(5, T, E).numpy()
    ids, w = oracle.route_topk(lg, k)
    rid, rw = _ref_route(lg, k)
    assert np.array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-14)
    assert np.all(np.abs(w.sum(1) - 1.0) <= 4.5e-16)


def test_route_ties_take_lower_id_and_minus_inf():
    lg = np.array([[0.5, 1.0, 1.0, -np.inf, 1.0, 0.2]], np.float32)
    ids, w = oracle.route_topk(lg, 3)
    assert list(ids[0]) == [1, 2, 4]
    assert np.allclose(w, 1 / 3, rtol=1e-15)
    z = synth.zipf_logits(0, 64, 256, 6).numpy()
    ids, w = oracle.route_topk(z, 6)
    for t in range(64):
        fin = np.nonzero(np.isfinite(z[t]))[0]
        assert set(ids[t]) == set(fin)
        np.testing.assert_allclose(w[t], softmax(z[t, ids[t]].astype(np.float64)), rtol=1e-14)


# ------------------------------------------------------------------ FP8 --

@pytest.mark.parametrize("b", [128, 32])
def test_fp8_block_linear_matches_library_formulation(b):
    """128x128 scale tiles (V4) and 32x32 (V4.1: "DeepSeek-V4.1-Flash mixed-Q2
    GGUF (IQ2_XXS gate/up + Q2_K down)", "Recipe")."""
    rng = np.random.default_rng(11)
    M, K, N = 3, 256, 384
    w = synth.fp8_codes(1, 7, N * K).numpy().reshape(N, K)
    s = rng.integers(118, 128, (N // b, K // b), dtype=np.uint8)
    x = synth.activations(4, M, K)
    y = oracle.fp8_block_linear(x, w, s, b)
    want = bf16_to_f64(x) @ dequant_fp8(w, s, b).astype(np.float64).T
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # one tile's scale moves only that tile's contribution
    s2 = s.copy()
    s2[1, 0] += 1
    y2 = oracle.fp8_block_linear(x, w, s2, b)
    assert np.array_equal(y2[:, :b], y[:, :b]) and np.array_equal(y2[:, 2 * b:], y[:, 2 * b:])
    assert not np.array_equal(y2[:, b:2 * b], y[:, b:2 * b])


@pytest.mark.parametrize("b", [128, 32])
def test_fp8_swiglu_ffn_matches_library_formulation(b):
    rng = np.random.default_rng(12)
    M, H, I = 2, 256, 128
    mats = []
    for t, (rows, cols) in enumerate(((I, H), (I, H), (H, I))):
        mats.append(synth.fp8_codes(2, t, rows * cols).numpy().reshape(rows, cols))
        mats.append(rng.integers(118, 128, (rows // b, cols // b), dtype=np.uint8))
    x = synth.activations(5, M, H)
    y = oracle.fp8_swiglu_ffn(x, *mats, block=b)
    x64 = bf16_to_f64(x)
    g = x64 @ dequant_fp8(mats[0], mats[1], b).astype(np.float64).T
    u = x64 @ dequant_fp8(mats[2], mats[3], b).astype(np.float64).T
    want = (g * expit(g) * u) @ dequant_fp8(mats[4], mats[5], b).astype(np.float64).T
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12 * np.abs(want).max())


def test_thread_count_does_not_change_results():
    E, H, I = 2, 256, 128
    ws = _layer(E, H, I, 118, 127, seed=13)
    x = synth.activations(6, 2, H)
    ids = np.array([[0, 1], [1, 0]], np.int32)
    w = np.array([[0.5, 0.5], [0.9, 0.1]])
    n0 = oracle.get_threads()
    oracle.set_threads(1)
    a = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    oracle.set_threads(max(2, n0))
    b = oracle.moe_forward(_oracle_layer(ws), x, ids, w)
    oracle.set_threads(n0)
    assert np.array_equal(a, b)
