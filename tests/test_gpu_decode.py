"""GPU parity of moe_expert_forward (decode path) against the oracle.

End to end from the same seeded logits: the GPU routes with moe_route_topk,
the oracle with its own softmax; the selected ids must agree exactly, then
y is compared with max|gpu - oracle| / max|oracle| <= 5e-3 and cosine >= 0.9999.
"""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import MX, NV, assert_parity, oracle_moe

pytestmark = pytest.mark.gpu


def _run(layer, x, ids, w, y_dtype=torch.float32):
    lay = layer.c()
    T, k = ids.shape
    y = torch.full((T, x.shape[1]), float("nan"), dtype=y_dtype, device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, T, k), dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x, ids, w, y, ws)
    assert qk.qk_last_device_status() == qk.QK_OK
    return y


def _e2e(wl, T, fmts, seed=0, layer_id=0, y_dtype=torch.float32, layer=None):
    layer = layer or workload.make_layer(wl, seed, layer_id, fmts)
    x = synth.activations(seed, T, wl.H, stream=layer_id)
    lg = synth.router_logits(seed, T, wl.E, stream=layer_id)
    ids = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    qk.moe_route_topk(lg.cuda(), wl.k, ids, w)
    y = _run(layer, x.cuda(), ids, w, y_dtype)
    oids, ow = oracle.route_topk(lg, wl.k)
    assert np.array_equal(ids.cpu().numpy(), oids)
    yo = oracle_moe(wl, seed, layer_id, x, oids, ow, fmts)
    return y.float().cpu().numpy(), yo


def test_tiny_config_mxfp4():
    wl = synth.WORKLOADS["tiny"]
    y, yo = _e2e(wl, wl.T, (MX, MX, MX))
    e, c = assert_parity(y, yo, what="tiny")
    assert e < 1e-3


@pytest.mark.parametrize("T", [1, 3, 8, 16])
def test_tiny_shapes_token_counts(T):
    wl = synth.WORKLOADS["tiny"]
    y, yo = _e2e(wl, T, (MX, MX, MX), seed=T)
    assert_parity(y, yo, what=f"tiny T={T}")


def test_decode_mxfp4_batch1_full_size():
    """Config C2: 256 experts, top-6, hidden 4096, intermediate 2048, 1 token."""
    wl = synth.WORKLOADS["decode_mx"]
    y, yo = _e2e(wl, 1, (MX, MX, MX))
    assert_parity(y, yo, what="decode_mx")


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_nvfp4_full_size(T):
    """Config C3: the same layer converted to NVFP4, batch 1, 4, 16."""
    wl = synth.WORKLOADS["decode_nv"]
    y, yo = _e2e(wl, T, (NV, NV, NV), seed=0)
    assert_parity(y, yo, what=f"decode_nv T={T}")


def test_nv_converted_equals_mx_output_closely():
    wl = synth.WORKLOADS["decode_mx"]
    mx = workload.make_layer(wl, 0, 0, (MX, MX, MX))
    nv = workload.DeviceLayer(*(workload.to_nvfp4(p) for p in (mx.gate, mx.up, mx.down)))
    x = synth.activations(3, 4, wl.H).cuda()
    ids = torch.tensor([[0, 5, 9, 77, 200, 255]] * 4, dtype=torch.int32, device="cuda")
    w = torch.full((4, 6), 1 / 6, device="cuda")
    a = _run(mx, x, ids, w).cpu().numpy()
    b = _run(nv, x, ids, w).cpu().numpy()
    # The conversion is lossless, so both layers hold the same weights.  The
    # MXFP4 layer runs on the block-scaled tensor cores (x exact as two e4m3
    # terms, h to 2^-12 as three); the NVFP4 layer on the f16 path (h rounded
    # to f16 after a row shift, 2^-11).  They differ by at most the two paths'
    # own errors against the exact result (about 2e-4 and 2e-5 measured).
    assert_parity(b, a, tol=5e-4, cos=0.9999999, what="nv vs mx")


@pytest.mark.parametrize("fmts", [(MX, NV, MX), (NV, MX, NV), (NV, NV, MX)])
def test_mixed_formats(fmts):
    wl = synth.Workload("mixed", 16, 4, 1024, 512, 5, 118, 127)
    y, yo = _e2e(wl, 5, fmts, seed=7)
    assert_parity(y, yo, what=f"mixed {fmts}")


def test_bf16_output():
    wl = synth.WORKLOADS["decode_mx"]
    y, yo = _e2e(wl, 2, (MX, MX, MX), seed=5, y_dtype=torch.bfloat16)
    assert_parity(y, yo, what="bf16 y")


def test_all_tokens_to_two_experts_token_tiles():
    """16 tokens all routed to experts 3 and 5: 16 tokens per expert exercises
    the multi-tile path; every other expert gets none."""
    wl = synth.Workload("hot", 8, 2, 512, 256, 16, 118, 127)
    layer = workload.make_layer(wl, 1, 0)
    x = synth.activations(1, 16, wl.H)
    ids = np.array([[3, 5]] * 16, np.int32)
    w = np.tile(np.array([[0.75, 0.25]]), (16, 1))
    y = _run(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda())
    yo = oracle_moe(wl, 1, 0, x, ids, w.astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy(), yo, what="hot experts")


def test_k1_single_expert_is_dense_ffn():
    wl = synth.Workload("k1", 4, 1, 256, 256, 3, 120, 127)
    layer = workload.make_layer(wl, 2, 0)
    x = synth.activations(2, 3, wl.H)
    ids = np.array([[2], [0], [2]], np.int32)
    w = np.ones((3, 1))
    y = _run(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.ones((3, 1), device="cuda"))
    assert_parity(y.cpu().numpy(), oracle_moe(wl, 2, 0, x, ids, w), what="k=1")


def test_deterministic_bytes():
    wl = synth.WORKLOADS["decode_nv"]
    layer = workload.make_layer(wl, 0, 0, (NV, NV, NV))
    x = synth.activations(9, 16, wl.H).cuda()
    lg = synth.router_logits(9, 16, wl.E).cuda()
    ids = torch.empty((16, 6), dtype=torch.int32, device="cuda")
    w = torch.empty((16, 6), device="cuda")
    qk.moe_route_topk(lg, 6, ids, w)
    a = _run(layer, x, ids, w)
    b = _run(layer, x, ids, w)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_large_activation_magnitudes():
    """Activations far outside f16 range are handled by the per-token shift."""
    wl = synth.WORKLOADS["tiny"]
    layer = workload.make_layer(wl, 0, 0)
    x = (synth.activations(4, 2, wl.H).float() * 2.0 ** 40).to(torch.bfloat16)
    x[1] *= 2.0 ** -80
    ids = np.array([[1, 6], [6, 2]], np.int32)
    w = np.array([[0.5, 0.5], [0.3, 0.7]])
    y = _run(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda())
    yo = oracle_moe(wl, 0, 0, x, ids, w.astype(np.float32).astype(np.float64))
    for t in range(2):
        assert_parity(y[t].cpu().numpy(), yo[t], what=f"scaled token {t}")


# ---- larger decode cases: random routing at mid size, full virtual experts,
# extreme activation magnitudes, determinism at full size ----

def test_mx_decode_random_routing_mid_size():
    """5 tokens, top-4 over 16 experts, hidden 1024, inter 1024 (the
    block-scaled decode path)."""
    wl = synth.Workload("mxmid", 16, 4, 1024, 1024, 5, 118, 127)
    y, yo = _e2e(wl, 5, (MX, MX, MX), seed=11)
    e, _ = assert_parity(y, yo, what="mx decode mid")
    assert e < 1e-4  # x exact as two e4m3 terms, h to 2^-12 as three


def test_mx_decode_full_virtual_experts():
    """16 tokens all routed to experts 3 and 12 (16 pairs each: two virtual
    experts of 8 pairs per expert), unequal weights."""
    wl = synth.Workload("mxhot", 16, 2, 1024, 1024, 16, 118, 127)
    layer = workload.make_layer(wl, 12, 0)
    x = synth.activations(12, 16, wl.H)
    ids = np.array([[3, 12]] * 16, np.int32)
    w = np.tile(np.array([[0.65, 0.35]]), (16, 1))
    y = _run(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda())
    yo = oracle_moe(wl, 12, 0, x, ids, w.astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy(), yo, what="mx hot experts")


def test_mx_decode_extreme_activations():
    """Token rows scaled by 2^40 and 2^-40: the per-32 ue8m0 scales of the
    activation terms follow each block's own range."""
    wl = synth.Workload("mxext", 16, 2, 1024, 1024, 2, 118, 127)
    layer = workload.make_layer(wl, 13, 0)
    x = synth.activations(13, 2, wl.H).float()
    x[0] *= 2.0 ** 40
    x[1] *= 2.0 ** -40
    x = x.to(torch.bfloat16)
    ids = np.array([[1, 9], [9, 4]], np.int32)
    w = np.array([[0.5, 0.5], [0.2, 0.8]])
    y = _run(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda())
    yo = oracle_moe(wl, 13, 0, x, ids, w.astype(np.float32).astype(np.float64))
    for t in range(2):
        assert_parity(y[t].cpu().numpy(), yo[t], what=f"mx extreme token {t}")


def test_mx_decode_deterministic():
    """MXFP4 at full size: the last unit of each output row tile forms y in
    slot order, so repeated calls give identical bytes."""
    wl = synth.WORKLOADS["decode_mx"]
    layer = workload.make_layer(wl, 0, 0)
    x = synth.activations(14, 3, wl.H).cuda()
    lg = synth.router_logits(14, 3, wl.E).cuda()
    ids = torch.empty((3, 6), dtype=torch.int32, device="cuda")
    w = torch.empty((3, 6), device="cuda")
    qk.moe_route_topk(lg, 6, ids, w)
    a = _run(layer, x, ids, w)
    b = _run(layer, x, ids, w)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
