"""moe_expert_forward_noalloc (scratch in the library's fixed device array)
against moe_expert_forward with a caller workspace, on the same inputs, two
calls in a row.  Collected last so it also runs after every other test."""
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import assert_parity

pytestmark = pytest.mark.gpu


def _inputs(wl, T, seed):
    layer = workload.make_layer(wl, seed, 0)
    x = synth.activations(seed, T, wl.H).cuda()
    lg = synth.router_logits(seed, T, wl.E).cuda()
    ids = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    qk.moe_route_topk(lg, wl.k, ids, w)
    return layer, x, ids, w


# decode_mx: the block-scaled decode kernels; decode_nv: the f16 decode
# kernels (NVFP4 layer); tiny at 100 tokens x top-2: the grouped path (200
# pairs, within the array for this small layer)
@pytest.mark.parametrize("name,T", [("decode_mx", 1), ("decode_mx", 4), ("tiny", 4), ("decode_nv", 4),
                                    ("tiny", 100)])
def test_noalloc_matches_workspace_entry(name, T):
    wl = synth.WORKLOADS[name]
    layer, x, ids, w = _inputs(wl, T, 3)
    lay = layer.c()
    ref = torch.empty((T, wl.H), dtype=torch.float32, device="cuda")
    ws = torch.empty(qk.moe_expert_workspace_size(lay, T, wl.k), dtype=torch.uint8, device="cuda")
    qk.moe_expert_forward(lay, x, ids, w, ref, ws)
    for call in range(2):
        y = torch.full_like(ref, float("nan"))
        qk.moe_expert_forward_noalloc(lay, x, ids, w, y)
        assert qk.qk_last_device_status() == qk.QK_OK
        assert_parity(y.cpu().numpy(), ref.cpu().numpy(), tol=1e-6, cos=0.999999,
                      what=f"noalloc call {call}")


def test_noalloc_rejects_requests_beyond_the_array():
    wl = synth.WORKLOADS["decode_mx"]
    layer, x, ids, w = _inputs(wl, 22, 4)  # 132 pairs: the grouped kernels, ~200 MB of scratch
    y = torch.empty((22, wl.H), dtype=torch.float32, device="cuda")
    with pytest.raises(qk.QkError) as e:
        qk.moe_expert_forward_noalloc(layer.c(), x, ids, w, y)
    assert e.value.code == qk.QK_ERR_WORKSPACE
