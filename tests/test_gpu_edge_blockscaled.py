"""Edge cases of the block-scaled MXFP4 kernels (decode and grouped paths)
against the oracle: e8m0 codes over a wide span (2^-40 .. 2^10), scale codes
0 and 254, all-zero weight blocks, activation blocks that are all zero or
bf16 subnormal, and the fp32 range limit.

Layers are drawn on the host (seeded generators), edited there, then copied
to the GPU; the oracle takes the same host bytes.  hidden 2048 and inter 1024
are multiples of 1024, so every MXFP4 layer here runs the block-scaled
kernels: up to floor(128 / top_k) tokens the decode kernels, above it the
grouped GEMMs.
"""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import MX, assert_parity

pytestmark = pytest.mark.gpu

WIDE = synth.Workload("edge_wide", 16, 4, 2048, 1024, 4, 87, 137)
BF16_MIN_NORMAL = 2.0 ** -126


def _host_layer(wl, seed):
    return workload.make_layer(wl, seed, 0, (MX, MX, MX), device="cpu")


def _dev(layer):
    return workload.DeviceLayer(*(workload.Proj(p.fmt, p.q.cuda(), p.scales.cuda())
                                  for p in (layer.gate, layer.up, layer.down)))


def _oracle_layer(layer):
    return oracle.Layer(*(oracle.Weight(MX, p.q.numpy(), p.scales.numpy())
                          for p in (layer.gate, layer.up, layer.down)))


def _bf16_bits(a):
    """float64 array -> bf16 bit patterns (uint16, round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16)


def _forward(dl, x_bits, ids, w):
    lay = dl.c()
    T, k = ids.shape
    y = torch.full((T, x_bits.shape[1]), float("nan"), device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, T, k), dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x_bits.cuda(), torch.from_numpy(ids).cuda(),
                          torch.from_numpy(w).float().cuda(), y, ws)
    st = qk.qk_last_device_status()
    return y.cpu().numpy(), st


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    lg = rng.standard_normal((T, k))
    w = np.exp(lg) / np.exp(lg).sum(1, keepdims=True)
    return ids, w


@pytest.mark.parametrize("T", [1, 3, 32, 40])
def test_wide_exponent_span(T):
    """e8m0 codes uniform over 87..137 (2^-40 .. 2^10) in all three projections;
    T = 1, 3, 32 run the decode kernels (top-4: up to 32 tokens), T = 40 the
    grouped GEMMs."""
    host = _host_layer(WIDE, 11)
    x = synth.activations(11, T, WIDE.H)
    ids, w = _routing(T, WIDE.E, WIDE.k, 11 + T)
    y, st = _forward(_dev(host), x, ids, w)
    assert st == qk.QK_OK
    yo = oracle.moe_forward(_oracle_layer(host), x, ids, w)
    assert_parity(y, yo, what=f"wide exponents T={T}")


def _edited(seed, T):
    """Scale codes 0 and 254, zero weight blocks, and activation blocks that are
    all zero, bf16 subnormal, or tiny (paired with code 254 so the products
    stay finite in fp32)."""
    wl = synth.Workload("edge_codes", 16, 4, 2048, 1024, T, 110, 130)
    host = _host_layer(wl, seed)
    g, u, d = host.gate, host.up, host.down
    ids, w = _routing(T, wl.E, wl.k, seed)
    e0 = int(ids[0, 0])
    x = synth.activations(seed, T, wl.H).view(torch.bfloat16).float().numpy().astype(np.float64)
    # gate: block 5 of rows 0..63 at 2^127 (code 254), x block 5 tiny (2^-120 scale)
    g.scales[e0, :64, 5] = 254
    x[:, 5 * 32:6 * 32] *= 2.0 ** -120
    # gate: whole rows 64..127 at code 0 (2^-127): their products underflow to ~0
    g.scales[e0, 64:128, :] = 0
    # up: rows 0..31, blocks 0..7 all-zero nibbles; down: block 3 of every row code 0
    u.q[e0, :32, :128] = 0
    d.scales[e0, :, 3] = 0
    # x: block 9 all zero, block 10 bf16 subnormal, block 11 spans 2^-60 .. 2^12
    x[:, 9 * 32:10 * 32] = 0.0
    x[:, 10 * 32:11 * 32] = np.linspace(-1, 1, 32) * BF16_MIN_NORMAL * 0.75
    x[:, 11 * 32:12 * 32] *= 2.0 ** np.linspace(-60, 12, 32)
    return host, _bf16_bits(x), ids, w


@pytest.mark.parametrize("T", [2, 40])
def test_scale_code_edges_zero_blocks_subnormal_x(T):
    host, xb, ids, w = _edited(21 + T, T)
    xs = xb.view(torch.bfloat16).float().numpy()
    assert np.any((xs != 0) & (np.abs(xs) < BF16_MIN_NORMAL)), "subnormal activations present"
    y, st = _forward(_dev(host), xb, ids, w)
    assert st == qk.QK_OK
    yo = oracle.moe_forward(_oracle_layer(host), xb, ids, w)
    assert_parity(y, yo, what=f"scale-code edges T={T}")


@pytest.mark.parametrize("T", [1, 40])
def test_fp32_overflow_reported(T):
    """A code-254 gate row against activations of ordinary size: the true
    gate value (about 2^130) lies beyond fp32, the fp64 oracle's does not.
    The kernels accumulate in fp32 (a documented range limit), detect the
    non-finite h and report QK_ERR_NONFINITE; tokens that do not route to the
    overflowing expert stay at parity."""
    wl = synth.Workload("edge_ovf", 16, 4, 2048, 1024, T, 118, 127)
    host = _host_layer(wl, 31)
    ids, w = _routing(T, wl.E, wl.k, 31)
    e0 = int(ids[0, 0])
    host.gate.scales[e0, 0, :] = 254
    x = synth.activations(31, T, wl.H)
    y, st = _forward(_dev(host), x, ids, w)
    assert st == qk.QK_ERR_NONFINITE
    yo = oracle.moe_forward(_oracle_layer(host), x, ids, w)
    assert np.isfinite(yo).all()
    clean = ~np.any(ids == e0, axis=1)
    if clean.any():
        assert np.isfinite(y[clean]).all()
        assert_parity(y[clean], yo[clean], what=f"overflow-free tokens T={T}")


@pytest.mark.parametrize("T", [1, 40])
def test_nonfinite_activation_reported(T):
    """An inf in x: the oracle's result is not finite; the kernels report
    QK_ERR_NONFINITE."""
    wl = synth.Workload("edge_inf", 16, 4, 2048, 1024, T, 118, 127)
    host = _host_layer(wl, 41)
    ids, w = _routing(T, wl.E, wl.k, 41)
    x = synth.activations(41, T, wl.H).view(torch.bfloat16).float().numpy().astype(np.float64)
    x[0, 100] = np.inf
    _, st = _forward(_dev(host), _bf16_bits(x), ids, w)
    assert st == qk.QK_ERR_NONFINITE
