"""GPU parity of moe_expert_forward at token counts beyond one launch's
routing capacity (consecutive launches over token slices), the 43-layer
stack's mixed-format decode layer, and the 2048-token Zipf prefill layer
(checked on sampled tokens; the oracle computes those tokens only).
"""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import MX, NV, assert_parity, oracle_moe

pytestmark = pytest.mark.gpu


def _forward(layer, x, ids, w, y_dtype=torch.float32):
    lay = layer.c()
    T, k = ids.shape
    y = torch.full((T, x.shape[1]), float("nan"), dtype=y_dtype, device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, T, k), dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x, ids, w, y, ws)
    assert qk.qk_last_device_status() == qk.QK_OK
    return y


@pytest.mark.parametrize("T", [65, 150])
def test_token_counts_beyond_one_launch(T):
    """Tiny layer, top-2: 64 tokens per launch, so 2 and 3 launches."""
    wl = synth.WORKLOADS["tiny"]
    layer = workload.make_layer(wl, T, 0)
    x = synth.activations(T, T, wl.H)
    lg = synth.router_logits(T, T, wl.E)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    yo = oracle_moe(wl, T, 0, x, oids, ow.astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy(), yo, what=f"tiny T={T}")


def test_stack_layer_mixed_formats():
    """One layer of the pruned 43-layer stack: 180 experts, top-6, 8 tokens,
    the seeded per-projection format choice of layer 5."""
    wl = synth.WORKLOADS["stack43"]
    fmts = tuple(int(f) for f in synth.format_choice(0, wl.layers)[5])
    layer = workload.make_layer(wl, 0, 5, fmts)
    x = synth.activations(0, wl.T, wl.H, stream=5)
    lg = synth.router_logits(0, wl.T, wl.E, stream=5)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    yo = oracle_moe(wl, 0, 5, x, oids, ow.astype(np.float32).astype(np.float64), fmts)
    assert_parity(y.cpu().numpy(), yo, what=f"stack layer 5 {fmts}")


@pytest.mark.parametrize("layer_id", [0, 17, 29, 42])
def test_stack_sampled_layers_with_shared_expert(layer_id):
    """The 43-layer stack on a seeded sample of its layers: 180 experts,
    top-6, 8 tokens, the layer's seeded per-projection formats, and the FP8
    block-128 shared expert added into the same output (y = routed + shared).
    The oracle regenerates both on the host.  The shared expert's synthetic
    FP8 weights (codes uniform over all 254 values) make its output about
    10^6 times the routed one, so each part is checked on its own as well as
    the sum."""
    wl = synth.WORKLOADS["stack43"]
    fmts = tuple(int(f) for f in synth.format_choice(0, wl.layers)[layer_id])
    layer = workload.make_layer(wl, 0, layer_id, fmts)
    sh = workload.make_fp8_shared(0, layer_id, wl.H, wl.I)
    x = synth.activations(0, wl.T, wl.H, stream=layer_id)
    lg = synth.router_logits(0, wl.T, wl.E, stream=layer_id)
    oids, ow = oracle.route_topk(lg, wl.k)
    xd = x.cuda()
    y = _forward(layer, xd, torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    y_routed = y.cpu().numpy().astype(np.float64)
    ws = torch.empty(qk.fp8_shared_expert_workspace_size(wl.T, wl.H, wl.I), dtype=torch.uint8,
                     device="cuda")
    qk.fp8_shared_expert_forward(xd, sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, y, ws)
    assert qk.qk_last_device_status() == qk.QK_OK
    y_total = y.cpu().numpy().astype(np.float64)
    ro = oracle_moe(wl, 0, layer_id, x, oids, ow.astype(np.float32).astype(np.float64), fmts)
    hs = workload.make_fp8_shared(0, layer_id, wl.H, wl.I, device="cpu")
    so = oracle.fp8_swiglu_ffn(x, hs.wg, hs.sg, hs.wu, hs.su, hs.wd, hs.sd)
    what = f"stack layer {layer_id} {fmts}"
    assert_parity(y_routed, ro, what=what + " routed")
    assert_parity(y_total - y_routed, so, what=what + " shared expert")
    assert_parity(y_total, ro + so, what=what + " routed + shared")


def _cover_tokens(oids, max_hot_bounds, seed):
    """Tokens that reach every expert's first and last token tile: each
    expert's first and last routed token (its pairs are grouped in token
    order, so these open and close its tile list), the tile boundaries of the
    hottest expert's list for both tile heights (40 and 64 tokens; evenly
    spaced, at most max_hot_bounds of them), and 10 random tokens."""
    T = oids.shape[0]
    first, last = {}, {}
    for t in range(T):
        for e in oids[t]:
            first.setdefault(int(e), t)
            last[int(e)] = t
    pick = set(first.values()) | set(last.values())
    counts = np.bincount(oids.reshape(-1))
    toks = np.nonzero((oids == int(np.argmax(counts))).any(1))[0]
    bounds = set()
    for tile in (40, 64):
        for b in range(0, len(toks), tile):
            bounds |= {int(toks[b]), int(toks[min(b + tile - 1, len(toks) - 1)])}
    bounds = sorted(bounds)
    if len(bounds) > max_hot_bounds:
        bounds = [bounds[i] for i in np.linspace(0, len(bounds) - 1, max_hot_bounds).round().astype(int)]
    pick |= set(bounds)
    pick |= set(int(t) for t in np.random.default_rng(seed).choice(T, 10, replace=False))
    return sorted(pick), len(first)


def test_prefill_zipf_sampled_tokens():
    """2048 tokens, Zipf-skewed routing over 256 experts, the bench's layer
    and routing: the tokens that open and close every expert's token tiles
    (so every expert group, its first and its last tile, and the tile
    boundaries of the hottest expert), about 380 of 2048, against the oracle."""
    wl = synth.WORKLOADS["prefill"]
    layer = workload.make_layer(wl, 0, 0)
    x = synth.activations(0, wl.T, wl.H)
    lg = synth.zipf_logits(0, wl.T, wl.E, wl.k)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    pick, n_exp = _cover_tokens(oids, 64, 7)
    assert n_exp == wl.E
    yo = oracle_moe(wl, 0, 0, x[pick], oids[pick], ow[pick].astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy()[pick], yo, what=f"prefill: {len(pick)} tokens covering every expert's tiles")


def test_prefill_16k_tokens_sampled():
    """The same prefill layer at 16,384 tokens (Zipf s=1, top-6, 256 experts,
    MXFP4: 98,304 pairs, past the size where the layer turns tensor-bound):
    every expert's first and last token and 32 tile boundaries spread over
    the hottest expert's ~11,000 pairs, against the oracle."""
    wl = synth.WORKLOADS["prefill"]
    T = 16384
    layer = workload.make_layer(wl, 0, 0)
    x = synth.activations(40, T, wl.H)
    oids, ow = oracle.route_topk(synth.zipf_logits(40, T, wl.E, wl.k), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    pick, n_exp = _cover_tokens(oids, 32, 41)
    assert n_exp == wl.E
    yo = oracle_moe(wl, 0, 0, x[pick], oids[pick], ow[pick].astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy()[pick], yo, what=f"prefill 16k: {len(pick)} tokens covering every expert")


@pytest.mark.parametrize("fmts", [(NV, NV, NV), (MX, NV, NV), (NV, MX, MX)])
def test_grouped_path_formats(fmts):
    """48 tokens x top-4 = 192 pairs (grouped path), NVFP4 and mixed projections."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, 48, 118, 127)
    layer = workload.make_layer(wl, 5, 0, fmts)
    x = synth.activations(5, wl.T, wl.H)
    lg = synth.router_logits(5, wl.T, wl.E)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    yo = oracle_moe(wl, 5, 0, x, oids, ow.astype(np.float32).astype(np.float64), fmts)
    assert_parity(y.cpu().numpy(), yo, what=f"grouped {fmts}")


def test_grouped_path_bf16_output_and_skewed_groups():
    """Tiny layer, 200 tokens all routed to experts 1 and 6 (groups of 200:
    a full and a partial token tile each); bf16 y."""
    wl = synth.WORKLOADS["tiny"]
    layer = workload.make_layer(wl, 6, 0)
    T = 200
    x = synth.activations(6, T, wl.H)
    ids = np.array([[1, 6]] * T, np.int32)
    w = np.tile(np.array([[0.6, 0.4]]), (T, 1))
    y = _forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda(),
                 torch.bfloat16)
    yo = oracle_moe(wl, 6, 0, x, ids, w.astype(np.float32).astype(np.float64))
    assert_parity(y.float().cpu().numpy(), yo, what="grouped bf16 y")


def test_mx_block_scaled_path():
    """All-MXFP4 layer with hidden and inter multiples of 512: the grouped
    path runs on the block-scaled tensor cores (e2m1 weights as stored, x as
    two e4m3 terms, h as three).  48 tokens x top-4 over 16 experts."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, 48, 118, 127)
    layer = workload.make_layer(wl, 8, 0)
    x = synth.activations(8, wl.T, wl.H)
    lg = synth.router_logits(8, wl.T, wl.E)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    yo = oracle_moe(wl, 8, 0, x, oids, ow.astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy(), yo, what="mx block-scaled")


def test_mx_path_skewed_groups_wide_exponents():
    """Block-scaled path, 300 tokens all routed to experts 1 and 6: three
    token tiles per expert (128, 128, 44 rows), one 512-element K chunk
    (hidden 512), e8m0 codes spanning 2^-40 .. 2^10, bf16 y."""
    wl = synth.Workload("wide", 8, 2, 512, 512, 300, 87, 137)
    layer = workload.make_layer(wl, 9, 0)
    x = synth.activations(9, wl.T, wl.H)
    ids = np.array([[1, 6]] * wl.T, np.int32)
    w = np.tile(np.array([[0.7, 0.3]]), (wl.T, 1))
    y = _forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).float().cuda(),
                 torch.bfloat16)
    yo = oracle_moe(wl, 9, 0, x, ids, w.astype(np.float32).astype(np.float64))
    assert_parity(y.float().cpu().numpy(), yo, what="mx skewed wide exponents")


def test_mx_path_many_small_groups():
    """Block-scaled path, 96 tokens x top-8 over 64 experts (groups of a few
    rows: 32-row token boxes), hidden 2048, inter 1024."""
    wl = synth.Workload("small_groups", 64, 8, 2048, 1024, 96, 118, 127)
    layer = workload.make_layer(wl, 10, 0)
    x = synth.activations(10, wl.T, wl.H)
    lg = synth.router_logits(10, wl.T, wl.E)
    oids, ow = oracle.route_topk(lg, wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda())
    yo = oracle_moe(wl, 10, 0, x, oids, ow.astype(np.float32).astype(np.float64))
    assert_parity(y.cpu().numpy(), yo, what="mx many small groups")
