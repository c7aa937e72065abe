"""GPU parity of the activation-quantized modes of moe_expert_forward:
QK_ACT_E4M3 (W4A8: fp4 weights x E4M3 activations, the numerics "DeepSeekv4
Flash for 1x Spark [REAP25]" (v0.2.3 update) names as the model's own) and
QK_ACT_MXFP4 (fp4 x fp4), against the oracle run in the same mode.

Both run on the grouped block-scaled kernels at every token count.  x codes
are unique on both sides (bf16 input); an h code may differ where fp32
rounding leaves it undetermined, which helpers.assert_parity_act_quant allows
for before applying the usual bar (max-rel <= 5e-3, cosine >= 0.9999)."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import MX, NV, assert_parity_act_quant, oracle_sublayer

pytestmark = pytest.mark.gpu

MODES = [qk.QK_ACT_E4M3, qk.QK_ACT_MXFP4]


def _forward(layer, x, ids, w, aq):
    lay = layer.c()
    T, k = ids.shape
    y = torch.full((T, x.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    n = qk.moe_expert_workspace_size(lay, T, k, aq)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x, ids, w, y, ws, act_quant=aq)
    assert qk.qk_last_device_status() == qk.QK_OK
    return y.cpu().numpy()


def _check(wl, seed, x, oids, ow, y, aq, what, fmts=(MX, MX, MX), nv_codes=None):
    """Parity in the mode, and a bound on the h codes taken from the other
    side of a decision boundary: an h value lies within the helper's relative
    window (2^-13) of a midpoint for well under 1 % of the codes (e4m3 steps
    are 2^-3 relative), so more than 0.5 % would mean a real difference, not
    rounding."""
    experts = sorted(set(int(e) for e in oids.reshape(-1)))
    remap = {e: i for i, e in enumerate(experts)}
    L = oracle_sublayer(wl, seed, 0, experts, fmts, nv_codes)
    sub = np.vectorize(remap.get)(oids).astype(np.int32)
    e, c, used, offered = assert_parity_act_quant(y, L, x, sub, ow.astype(np.float32).astype(np.float64), aq,
                                                  what=what)
    n_codes = oids.size * wl.I
    assert used <= offered and used <= max(8, n_codes // 200), (what, used, offered, n_codes)
    return e, c, used, offered


@pytest.mark.parametrize("aq", MODES)
@pytest.mark.parametrize("T", [1, 4])
def test_decode_sizes(aq, T):
    """The decode MoE layer (256 experts, top-6, hidden 4096, intermediate
    2048, MXFP4) at 1 and 4 tokens."""
    wl = synth.WORKLOADS["decode_mx"]
    layer = workload.make_layer(wl, 21, 0)
    x = synth.activations(21, T, wl.H)
    oids, ow = oracle.route_topk(synth.router_logits(21, T, wl.E), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(), aq)
    _check(wl, 21, x, oids, ow, y, aq, f"act mode {aq} decode T={T}")


@pytest.mark.parametrize("aq", MODES)
def test_grouped_sizes(aq):
    """48 tokens x top-4 over 16 experts, hidden 1024, intermediate 512."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, 48, 118, 127)
    layer = workload.make_layer(wl, 22, 0)
    x = synth.activations(22, wl.T, wl.H)
    oids, ow = oracle.route_topk(synth.router_logits(22, wl.T, wl.E), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(), aq)
    _check(wl, 22, x, oids, ow, y, aq, f"act mode {aq} grouped")


def test_w4a8_prefill_zipf_sampled_tokens():
    """The 2048-token Zipf prefill layer in W4A8: the tokens that open and
    close every expert's token tiles, and 10 random ones."""
    wl = synth.WORKLOADS["prefill"]
    layer = workload.make_layer(wl, 23, 0)
    x = synth.activations(23, wl.T, wl.H)
    oids, ow = oracle.route_topk(synth.zipf_logits(23, wl.T, wl.E, wl.k), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(),
                 qk.QK_ACT_E4M3)
    # every expert's first and last token (the first and last tile of each
    # expert group) and 10 random tokens
    first, last = {}, {}
    for t in range(wl.T):
        for e in oids[t]:
            first.setdefault(int(e), t)
            last[int(e)] = t
    pick = set(first.values()) | set(last.values())
    pick |= set(int(t) for t in np.random.default_rng(24).choice(wl.T, 10, replace=False))
    pick = sorted(pick)
    _check(wl, 23, x[pick], oids[pick], ow[pick], y[pick], qk.QK_ACT_E4M3,
           f"w4a8 prefill: {len(pick)} tokens covering every expert")


def test_w4a4_prefill_zipf_sampled_tokens():
    """The 2048-token Zipf prefill layer with QK_ACT_MXFP4 (fp4 x fp4:
    kind::mxf4 on 128-token tiles, the hottest expert's group spanning about
    eleven of them): the tokens that open and close every expert's token
    tiles, and 10 random ones."""
    wl = synth.WORKLOADS["prefill"]
    layer = workload.make_layer(wl, 26, 0)
    x = synth.activations(26, wl.T, wl.H)
    oids, ow = oracle.route_topk(synth.zipf_logits(26, wl.T, wl.E, wl.k), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(),
                 qk.QK_ACT_MXFP4)
    first, last = {}, {}
    for t in range(wl.T):
        for e in oids[t]:
            first.setdefault(int(e), t)
            last[int(e)] = t
    counts = np.bincount(oids.reshape(-1))
    hot = np.nonzero((oids == int(np.argmax(counts))).any(1))[0]
    pick = set(first.values()) | set(last.values()) | set(int(t) for t in hot[127::128]) | set(int(t) for t in hot[128::128])
    pick |= set(int(t) for t in np.random.default_rng(27).choice(wl.T, 10, replace=False))
    pick = sorted(pick)
    _check(wl, 26, x[pick], oids[pick], ow[pick], y[pick], qk.QK_ACT_MXFP4,
           f"w4a4 prefill: {len(pick)} tokens covering every expert")


# NVFP4 layers in QK_ACT_MXFP4 run fp4 x fp4 on kind::mxf4nvf4: converted
# from MXFP4 (power-of-two block scales and scale_2), and general (any e4m3
# block scale, scale_2 not a power of two).
NV_SOURCES = [None, (synth.NV_CODE_LO, synth.NV_CODE_HI)]


@pytest.mark.parametrize("codes", NV_SOURCES, ids=["converted", "general"])
@pytest.mark.parametrize("T", [1, 48])
def test_nvfp4_w4a4_mxf4nvf4(codes, T):
    """48 tokens (or 1) x top-4 over 16 experts, hidden 1024, intermediate 512,
    all three projections NVFP4."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, T, 118, 127)
    layer = workload.make_layer(wl, 31, 0, (NV, NV, NV), nv_codes=codes)
    x = synth.activations(31, T, wl.H)
    oids, ow = oracle.route_topk(synth.router_logits(31, T, wl.E), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(),
                 qk.QK_ACT_MXFP4)
    _check(wl, 31, x, oids, ow, y, qk.QK_ACT_MXFP4, f"nvfp4 w4a4 T={T} {'general' if codes else 'converted'}",
           (NV, NV, NV), codes)


def test_nvfp4_w4a4_decode_layer():
    """The decode MoE layer in NVFP4 (256 experts, top-6, hidden 4096,
    intermediate 2048, converted from the seeded MXFP4 layer) at 4 tokens."""
    wl = synth.WORKLOADS["decode_mx"]
    layer = workload.make_layer(wl, 32, 0, (NV, NV, NV))
    x = synth.activations(32, 4, wl.H)
    oids, ow = oracle.route_topk(synth.router_logits(32, 4, wl.E), wl.k)
    y = _forward(layer, x.cuda(), torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda(),
                 qk.QK_ACT_MXFP4)
    _check(wl, 32, x, oids, ow, y, qk.QK_ACT_MXFP4, "nvfp4 w4a4 decode layer T=4", (NV, NV, NV))


def test_nvfp4_w4a8_refused():
    """W4A8 has no NVFP4 form on sm_100a: kind::mxf8f6f4 takes ue8m0 scales
    only, so an NVFP4 layer in QK_ACT_E4M3 is refused (workspace 0)."""
    wl = synth.Workload("mid", 16, 4, 1024, 512, 4, 118, 127)
    lay = workload.make_layer(wl, 33, 0, (NV, NV, NV)).c()
    assert qk.moe_expert_workspace_size(lay, 4, 4, qk.QK_ACT_E4M3) == 0
    assert qk.moe_expert_workspace_size(lay, 4, 4, qk.QK_ACT_MXFP4) > 0


@pytest.mark.parametrize("aq", MODES)
def test_modes_are_deterministic_and_differ_from_bf16(aq):
    wl = synth.Workload("mid", 16, 4, 1024, 512, 24, 118, 127)
    layer = workload.make_layer(wl, 25, 0)
    x = synth.activations(25, wl.T, wl.H).cuda()
    oids, ow = oracle.route_topk(synth.router_logits(25, wl.T, wl.E), wl.k)
    ids, w = torch.from_numpy(oids).cuda(), torch.from_numpy(ow).float().cuda()
    a = _forward(layer, x, ids, w, aq)
    b = _forward(layer, x, ids, w, aq)
    assert np.array_equal(a.view(np.int32), b.view(np.int32))
    plain = _forward(layer, x, ids, w, qk.QK_ACT_NONE)
    assert not np.array_equal(a, plain)
