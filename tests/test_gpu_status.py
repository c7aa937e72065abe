"""Device-detected errors: NaN scale codes, expert ids out of range, and the
bounded-wait timeout path (forced by a zero wait limit; nothing hangs)."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import assert_parity, oracle_moe

pytestmark = pytest.mark.gpu

WL = synth.Workload("small", 8, 2, 256, 256, 4, 118, 127)
# hidden 2048, inter 1024: multiples of 1024, so MXFP4 layers take the
# block-scaled kernels (decode up to floor(128 / top_k) = 32 tokens, grouped
# GEMMs above)
BS = synth.Workload("bs_status", 16, 4, 2048, 1024, 4, 118, 127)


def _setup(seed=0):
    layer = workload.make_layer(WL, seed, 0)
    x = synth.activations(seed, WL.T, WL.H)
    return layer, x


def _fwd(layer, x, ids, w):
    lay = layer.c()
    y = torch.zeros((x.shape[0], WL.H), device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, x.shape[0], ids.shape[1]),
                     dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x.cuda(), ids, w, y, ws)
    return y


def test_nan_scale_reported():
    layer, x = _setup()
    layer.up.scales[2, 7, 3] = 255
    ids = torch.tensor([[2, 1]] * 4, dtype=torch.int32, device="cuda")
    w = torch.full((4, 2), 0.5, device="cuda")
    _fwd(layer, x, ids, w)
    assert qk.qk_last_device_status() == qk.QK_ERR_NAN_SCALE


def test_nan_e4m3_block_scale_reported_decode():
    """NVFP4 (a general source): e4m3 0x7F in one block scale, decode path."""
    layer = workload.make_layer(WL, 3, 0, (2, 2, 2), nv_codes=(0x60, 0x7E))
    layer.up.scales[2, 7, 5] = 0x7F
    x = synth.activations(3, WL.T, WL.H)
    ids = torch.tensor([[2, 1]] * 4, dtype=torch.int32, device="cuda")
    w = torch.full((4, 2), 0.5, device="cuda")
    _fwd(layer, x, ids, w)
    assert qk.qk_last_device_status() == qk.QK_ERR_NAN_SCALE


@pytest.mark.parametrize("fmt,code", [(1, 0xFF), (2, 0x7F), (2, 0xFF)])
def test_nan_scale_reported_grouped(fmt, code):
    """100 tokens x top-2 (the grouped GEMMs): one NaN scale code in expert
    2's up projection (e8m0 0xFF; e4m3 0x7F or 0xFF)."""
    layer = workload.make_layer(WL, 4, 0, (fmt, fmt, fmt), nv_codes=(0x60, 0x7E))
    layer.up.scales[2, 7, 3] = code
    x = synth.activations(4, 100, WL.H)
    ids = torch.tensor([[2, 1]] * 100, dtype=torch.int32, device="cuda")
    w = torch.full((100, 2), 0.5, device="cuda")
    _fwd(layer, x, ids, w)
    assert qk.qk_last_device_status() == qk.QK_ERR_NAN_SCALE


def test_out_of_range_id_reported_and_skipped():
    layer, x = _setup(1)
    ids_np = np.array([[1, 4], [8, 2], [3, -1], [0, 7]], np.int32)
    w_np = np.full((4, 2), 0.5)
    y = _fwd(layer, x, torch.from_numpy(ids_np).cuda(), torch.from_numpy(w_np).float().cuda())
    assert qk.qk_last_device_status() == qk.QK_ERR_INVALID_ARG
    valid = (ids_np >= 0) & (ids_np < WL.E)
    w_eff = np.where(valid, w_np, 0.0)
    ids_eff = np.where(valid, ids_np, 0).astype(np.int32)
    yo = oracle_moe(WL, 1, 0, x, ids_eff, w_eff)
    assert_parity(y.cpu().numpy(), yo, what="skipped pairs")


def _fwd_wl(wl, layer, x, ids, w):
    lay = layer.c()
    y = torch.zeros((x.shape[0], wl.H), device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, x.shape[0], ids.shape[1]),
                     dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x.cuda(), ids, w, y, ws)
    return y


def _timeout_then_parity(wl, layer, seed, x, ids_np, w_np, what, fmts=(1, 1, 1)):
    """Three calls with the wait limit at 0 (the first wait not already
    complete runs out: weight copies take about a microsecond to land, so at
    least one does), then a call at the default limit checked against the
    oracle: the kernels stop cleanly and the context stays usable."""
    ids = torch.from_numpy(ids_np).cuda()
    w = torch.from_numpy(w_np).float().cuda()
    seen = []
    try:
        qk.qk_debug_set_wait_limit_ns(0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        for i in range(3):
            flush.fill_(i)  # the weights leave L2: the first copies cannot have landed at the first poll
            _fwd_wl(wl, layer, x, ids, w)
            seen.append(qk.qk_last_device_status())
    finally:
        qk.qk_debug_set_wait_limit_ns(1_000_000_000)
    assert qk.QK_ERR_TIMEOUT in seen, seen
    assert all(s in (qk.QK_ERR_TIMEOUT, qk.QK_OK) for s in seen), seen
    y = _fwd_wl(wl, layer, x, ids, w)
    assert qk.qk_last_device_status() == qk.QK_OK
    yo = oracle_moe(wl, seed, 0, x, ids_np, w_np, fmts)
    assert_parity(y.cpu().numpy(), yo, what=what)


def test_timeout_path_reports_and_context_survives():
    """The f16 decode kernels: the full-size NVFP4 decode layer (256 experts,
    hidden 4096, inter 2048; the block-scaled decode takes MXFP4 layers only)
    at one token, its weights out of L2 before each call."""
    wl = synth.WORKLOADS["decode_nv"]
    layer = workload.make_layer(wl, 2, 0, (2, 2, 2))
    x = synth.activations(2, 1, wl.H)
    ids = np.array([[3, 17, 40, 99, 150, 201]], np.int32)
    w = np.full((1, 6), 1.0 / 6)
    _timeout_then_parity(wl, layer, 2, x, ids, w, "f16 decode after timeout", fmts=(2, 2, 2))


def _bs_routing(T, seed):
    """Slot 0 of every token is expert 3; the other slots are distinct random
    experts."""
    rng = np.random.default_rng(seed)
    others = [e for e in range(BS.E) if e != 3]
    ids = np.array([[3] + list(rng.choice(others, size=BS.k - 1, replace=False)) for _ in range(T)],
                   dtype=np.int32)
    w = np.full((T, BS.k), 1.0 / BS.k)
    return ids, w


@pytest.mark.parametrize("T", [2, 40])
def test_timeout_block_scaled(T):
    """Block-scaled MXFP4 kernels: T = 2 runs the decode kernels, T = 40 (160
    pairs) the grouped GEMMs; every wait there is bounded and reports."""
    layer = workload.make_layer(BS, 6, 0)
    x = synth.activations(6, T, BS.H)
    ids, w = _bs_routing(T, 6 + T)
    _timeout_then_parity(BS, layer, 6, x, ids, w, f"block-scaled T={T} after timeout")


@pytest.mark.parametrize("T", [2, 40])
def test_nan_scale_reported_block_scaled(T):
    """e8m0 code 255 in expert 3's up projection, block-scaled decode (T = 2)
    and grouped (T = 40) kernels."""
    layer = workload.make_layer(BS, 7, 0)
    layer.up.scales[3, 7, 2] = 255
    x = synth.activations(7, T, BS.H)
    ids, w = _bs_routing(T, 7 + T)
    _fwd_wl(BS, layer, x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda())
    assert qk.qk_last_device_status() == qk.QK_ERR_NAN_SCALE


@pytest.mark.parametrize("code", [0x7F, 0xFF])
def test_nan_e4m3_scale_reported_nvfp4_fp4_mode(code):
    """An NVFP4 layer in QK_ACT_MXFP4 (the kind::mxf4nvf4 grouped kernels,
    whose weight-scale warp checks e4m3 NaN codes 0x7F and 0xFF): one NaN
    block scale in expert 3's up projection, 4 tokens."""
    layer = workload.make_layer(BS, 8, 0, (2, 2, 2), nv_codes=(0x60, 0x7E))
    layer.up.scales[3, 7, 2] = code
    x = synth.activations(8, 4, BS.H)
    ids, w = _bs_routing(4, 15)
    lay = layer.c()
    y = torch.zeros((4, BS.H), device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, 4, BS.k, qk.QK_ACT_MXFP4), dtype=torch.uint8,
                     device="cuda")
    qk.moe_expert_forward(lay, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda(), y, ws,
                          act_quant=qk.QK_ACT_MXFP4)
    assert qk.qk_last_device_status() == qk.QK_ERR_NAN_SCALE
