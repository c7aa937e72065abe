"""GPU parity: softmax top-k router.  ids bit-exact, weights within 1e-6."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth

pytestmark = pytest.mark.gpu


def _route(lg, k):
    T, E = lg.shape
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    qk.moe_route_topk(lg.cuda(), k, ids, w)
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,k", [(4, 8, 2), (1, 256, 6), (16, 256, 6), (8, 180, 6),
                                   (33, 2048, 32), (2048, 256, 6)])
def test_route_matches_oracle(T, E, k):
    lg = synth.router_logits(T + E, T, E)
    ids, w = _route(lg, k)
    oids, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids, oids)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)
    assert qk.qk_last_device_status() == qk.QK_OK


def test_route_ties_and_minus_inf():
    lg = torch.tensor([[0.5, 1.0, 1.0, -np.inf, 1.0, 0.2]], dtype=torch.float32)
    ids, w = _route(lg, 3)
    assert list(ids[0]) == [1, 2, 4]
    z = synth.zipf_logits(0, 2048, 256, 6)
    ids, w = _route(z, 6)
    oids, ow = oracle.route_topk(z, 6)
    assert np.array_equal(ids, oids)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)


def test_route_all_minus_inf_sets_status():
    lg = torch.full((2, 8), -np.inf)
    _route(lg, 2)
    assert qk.qk_last_device_status() == qk.QK_ERR_INVALID_ARG
