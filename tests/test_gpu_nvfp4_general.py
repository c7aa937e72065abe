"""GPU parity of moe_expert_forward on general NVFP4 sources: e4m3 block
scales and a per-expert fp32 scale_2 that are not powers of two (an NVFP4
checkpoint quantized directly, not converted from MXFP4).

The format ("DeepSeek-v4-Flash-REAP-K180-NVFP4", section "NVFP4: lossless
MXFP4->NVFP4 conversion") admits any non-NaN e4m3 block scale and any fp32
scale_2; both NVFP4 kernel paths (decode: k_decode, grouped: k_ggemm) take
e2m1 x e4m3 exactly in f16 and apply scale_2 to the fp32 result.  Same bar as
every other parity test: max|gpu - oracle| / max|oracle| <= 5e-3 and cosine
>= 0.9999, against the oracle's exact (fp64) dequantization.
"""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import MX, NV, assert_parity, oracle_moe

pytestmark = pytest.mark.gpu

GENERAL = (synth.NV_CODE_LO, synth.NV_CODE_HI)  # e4m3 32 .. 448, every mantissa
ALL_CODES = (0x00, 0x7E)                        # zero, subnormal and normal block scales


def _forward(layer, x, ids, w):
    lay = layer.c()
    T, k = ids.shape
    y = torch.full((T, x.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, T, k), dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x, ids, w, y, ws)
    assert qk.qk_last_device_status() == qk.QK_OK
    return y.cpu().numpy()


def _e2e(wl, T, fmts, codes, seed, route_on_gpu=True):
    layer = workload.make_layer(wl, seed, 0, fmts, nv_codes=codes)
    assert all(p.fmt == f for p, f in zip((layer.gate, layer.up, layer.down), fmts))
    x = synth.activations(seed, T, wl.H)
    lg = synth.router_logits(seed, T, wl.E)
    oids, ow = oracle.route_topk(lg, wl.k)
    if route_on_gpu:  # the GPU routes itself; the oracle keeps its own weights
        ids = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
        qk.moe_route_topk(lg.cuda(), wl.k, ids, w)
        assert np.array_equal(ids.cpu().numpy(), oids)
    else:  # both sides take the oracle's routing, the GPU its fp32 weights
        ids = torch.from_numpy(oids).cuda()
        w = torch.from_numpy(ow).float().cuda()
        ow = ow.astype(np.float32).astype(np.float64)
    y = _forward(layer, x.cuda(), ids, w)
    yo = oracle_moe(wl, seed, 0, x, oids, ow, fmts, codes)
    return y, yo


def test_tiny_every_block_scale_code_decode():
    wl = synth.WORKLOADS["tiny"]
    y, yo = _e2e(wl, wl.T, (NV, NV, NV), ALL_CODES, seed=11)
    assert_parity(y, yo, what="general nv tiny, all codes (decode)")


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_full_size(T):
    """256 experts, top-6, hidden 4096, intermediate 2048, general NVFP4."""
    wl = synth.WORKLOADS["decode_nv"]
    y, yo = _e2e(wl, T, (NV, NV, NV), GENERAL, seed=12)
    assert_parity(y, yo, what=f"general nv decode T={T}")


@pytest.mark.parametrize("fmts", [(MX, NV, MX), (NV, MX, NV)])
def test_mixed_with_mxfp4_decode(fmts):
    wl = synth.Workload("mixed", 16, 4, 1024, 512, 5, 118, 127)
    y, yo = _e2e(wl, 5, fmts, GENERAL, seed=13)
    assert_parity(y, yo, what=f"general nv mixed {fmts} (decode)")


@pytest.mark.parametrize("fmts", [(NV, NV, NV), (MX, NV, NV), (NV, MX, MX)])
def test_grouped_path(fmts):
    """48 tokens x top-4 = 192 pairs over 16 experts: the grouped GEMMs."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, 48, 118, 127)
    y, yo = _e2e(wl, 48, fmts, GENERAL, seed=14, route_on_gpu=False)
    assert_parity(y, yo, what=f"general nv grouped {fmts}")


def test_grouped_every_block_scale_code():
    """Tiny layer, 200 tokens (grouped path), block scales over every
    non-NaN positive e4m3 code."""
    wl = synth.WORKLOADS["tiny"]
    y, yo = _e2e(wl, 200, (NV, NV, NV), ALL_CODES, seed=15, route_on_gpu=False)
    assert_parity(y, yo, what="general nv tiny, all codes (grouped)")


def test_prefill_zipf_sampled_tokens():
    """The 2048-token Zipf prefill layer with general NVFP4 weights (grouped
    f16 GEMMs); 12 sampled tokens, including ones routed to the most and the
    least loaded experts, against the oracle."""
    wl = synth.WORKLOADS["prefill"]
    layer = workload.make_layer(wl, 16, 0, (NV, NV, NV), nv_codes=GENERAL)
    x = synth.activations(16, wl.T, wl.H)
    lg = synth.zipf_logits(16, wl.T, wl.E, wl.k)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    counts = np.bincount(oids.reshape(-1), minlength=wl.E)
    hot, cold = int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    pick = {int(np.nonzero((oids == hot).any(1))[0][0]), int(np.nonzero((oids == cold).any(1))[0][0])}
    pick |= set(int(t) for t in np.random.default_rng(17).choice(wl.T, 10, replace=False))
    pick = sorted(pick)
    yo = oracle_moe(wl, 16, 0, x[pick], oids[pick], ow[pick].astype(np.float32).astype(np.float64),
                    (NV, NV, NV), GENERAL)
    assert_parity(y[pick], yo, what="general nv prefill sampled tokens")
