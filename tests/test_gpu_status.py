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


def test_timeout_path_reports_and_context_survives():
    layer, x = _setup(2)
    ids = torch.tensor([[0, 1]] * 4, dtype=torch.int32, device="cuda")
    w = torch.full((4, 2), 0.5, device="cuda")
    try:
        qk.qk_debug_set_wait_limit_ns(0)
        for _ in range(3):
            _fwd(layer, x, ids, w)
        st = qk.qk_last_device_status()
    finally:
        qk.qk_debug_set_wait_limit_ns(1_000_000_000)
    assert st in (qk.QK_ERR_TIMEOUT, qk.QK_OK)  # a copy may land before the first poll
    y = _fwd(layer, x, ids, w)
    assert qk.qk_last_device_status() == qk.QK_OK
    yo = oracle_moe(WL, 2, 0, x, np.array([[0, 1]] * 4, np.int32), np.full((4, 2), 0.5))
    assert_parity(y.cpu().numpy(), yo, what="after timeout")
