"""GPU parity: scale-only NVFP4 -> MXFP4 conversion (the reverse direction,
exact where possible), bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth

pytestmark = pytest.mark.gpu


def _gpu_reverse(e4_np, s2_np):
    e4 = torch.from_numpy(np.ascontiguousarray(e4_np)).cuda()
    s2 = torch.from_numpy(np.ascontiguousarray(s2_np, np.float32)).cuda()
    E, N, K16 = e4.shape
    out = torch.full((E, N, K16 // 2), 0xAA, dtype=torch.uint8, device="cuda")
    bad = torch.full((1,), 12345, dtype=torch.int64, device="cuda")
    qk.quant_convert_nvfp4_to_mxfp4(e4, s2, out, bad)
    st = qk.qk_last_device_status()
    return out.cpu().numpy(), int(bad.item()), st


@pytest.mark.parametrize("E,N,K,codes", [
    (4, 64, 512, (0x60, 0x7E)),   # general sources: almost every block inexact
    (3, 5, 96, (0x00, 0x7E)),     # every positive code, odd block count per expert
    (2, 1, 32, (0x38, 0x38)),     # one block per expert, equal halves
])
def test_general_sources_match_oracle(E, N, K, codes):
    _, e4, s2 = synth.nv_expert_bytes(31, 0, 0, N, K, None, E, "cpu", *codes)
    e4, s2 = e4.numpy(), s2.numpy()
    out, bad, st = _gpu_reverse(e4, s2)
    want, wbad = oracle.convert_nv_to_mx(e4, s2)
    assert st == qk.QK_OK
    assert np.array_equal(out, want) and bad == wbad


def test_edge_scales_match_oracle():
    rng = np.random.default_rng(32)
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    e4 = codes[rng.integers(0, codes.size, (6, 40, 64))]
    e4[:, :10] = 0x38                                   # equal power-of-two halves
    s2 = np.array([1.0, 2.0 ** -9, 2.0 ** -130, 3.0e38, -0.5, 0.1], np.float32)
    out, bad, st = _gpu_reverse(e4, s2)
    want, wbad = oracle.convert_nv_to_mx(e4, s2)
    assert st == qk.QK_OK
    assert np.array_equal(out, want) and bad == wbad


def test_round_trip_of_a_full_projection_is_the_identity():
    """The decode layer's gate projection (256 experts x 2048 rows x 4096):
    MXFP4 -> NVFP4 -> MXFP4 on the GPU returns the original codes."""
    wl = synth.WORKLOADS["decode_mx"]
    _, s = synth.mx_expert_bytes(0, 0, synth.TID.GATE, wl.I, wl.H, wl.code_lo, wl.code_hi, None, wl.E,
                                 "cuda")
    E, N, K32 = s.shape
    e4 = torch.empty((E, N, 2 * K32), dtype=torch.uint8, device="cuda")
    s2 = torch.empty(E, dtype=torch.float32, device="cuda")
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    qk.quant_convert_mxfp4_to_nvfp4(s, e4, s2, bad)
    assert int(bad.item()) == 0
    back = torch.empty_like(s)
    qk.quant_convert_nvfp4_to_mxfp4(e4, s2, back, bad)
    assert qk.qk_last_device_status() == qk.QK_OK
    assert int(bad.item()) == 0 and torch.equal(back, s)


def test_nan_code_sets_status_and_writes_255():
    e4 = np.full((1, 2, 4), 0x38, np.uint8)
    e4[0, 1, 3] = 0x7F
    out, bad, st = _gpu_reverse(e4, np.ones(1, np.float32))
    assert st == qk.QK_ERR_NAN_SCALE
    assert out[0, 1, 1] == 255 and out[0, 0, 0] == 127 and out[0, 1, 0] == 127
