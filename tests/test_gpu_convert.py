"""GPU parity: scale-only MXFP4 -> NVFP4 conversion, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth

pytestmark = pytest.mark.gpu


def _gpu_convert(s_np):
    s = torch.from_numpy(np.ascontiguousarray(s_np)).cuda()
    E, N, K32 = s.shape
    e4 = torch.full((E, N, 2 * K32), 0xAA, dtype=torch.uint8, device="cuda")
    s2 = torch.empty(E, dtype=torch.float32, device="cuda")
    bad = torch.full((1,), 12345, dtype=torch.int64, device="cuda")
    qk.quant_convert_mxfp4_to_nvfp4(s, e4, s2, bad)
    st = qk.qk_last_device_status()
    return e4.cpu().numpy(), s2.cpu().numpy(), int(bad.item()), st


def _check(s_np):
    e4, s2, bad, st = _gpu_convert(s_np)
    oe4, os2, obad = oracle.convert_mx_to_nv(s_np)
    assert st == qk.QK_OK
    assert np.array_equal(e4, oe4)
    assert np.array_equal(s2.view(np.uint32), os2.view(np.uint32))
    assert bad == obad
    return bad


@pytest.mark.parametrize("E,N,K,lo,hi", [
    (8, 128, 256, 121, 129),      # tiny config's projections
    (3, 5, 96, 118, 127),         # per = 15: unaligned scalar path
    (4, 7, 64, 0, 254),           # full code range: inexact blocks
    (2, 1, 32, 200, 200),         # one block per expert
    (16, 64, 4096, 118, 127),
])
def test_convert_matches_oracle(E, N, K, lo, hi):
    rng = np.random.default_rng(E * 1000 + N)
    s = rng.integers(lo, hi + 1, (E, N, K // 32), dtype=np.uint8)
    _check(s)


def test_convert_full_layer_projection_bit_exact():
    """A full decode-layer projection: 256 experts x 2048 x 4096 (config C3)."""
    wl = synth.WORKLOADS["decode_nv"]
    s = synth.scale_codes(0, synth.TID.of(0, synth.TID.GATE, synth.TID.SCALES),
                          wl.E * wl.I * wl.H // 32, wl.code_lo, wl.code_hi, "cuda")
    s = s.view(wl.E, wl.I, wl.H // 32)
    e4 = torch.empty((wl.E, wl.I, wl.H // 16), dtype=torch.uint8, device="cuda")
    s2 = torch.empty(wl.E, dtype=torch.float32, device="cuda")
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    qk.quant_convert_mxfp4_to_nvfp4(s, e4, s2, bad)
    oe4, os2, obad = oracle.convert_mx_to_nv(s.cpu().numpy())
    assert np.array_equal(e4.cpu().numpy(), oe4)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), os2.view(np.uint32))
    assert int(bad.item()) == obad == 0
    # deterministic: a second run gives the same bytes
    e4b = torch.empty_like(e4)
    qk.quant_convert_mxfp4_to_nvfp4(s, e4b, s2, bad)
    assert torch.equal(e4, e4b)


def test_span_edges_and_extremes():
    s = np.full((3, 2, 4), 150, np.uint8)
    s[0, 0, 1] = 150 - 17          # exact
    s[1, 1, 3] = 150 - 18          # 2^-10 -> 0
    s[1, 0, 0] = 150 - 40          # -> 0
    s[2] = 0                       # all code 0: scale_2 = 2^-135 (subnormal)
    assert _check(s) == 2


def test_nan_code_sets_status_and_nan_output():
    s = np.full((2, 2, 2), 120, np.uint8)
    s[1, 0, 1] = 255
    e4, s2, bad, st = _gpu_convert(s)
    assert st == qk.QK_ERR_NAN_SCALE
    assert e4[1, 0, 2] == 0x7F and e4[1, 0, 3] == 0x7F
    assert qk.qk_last_device_status() == qk.QK_OK  # read clears


def test_nibbles_untouched_and_dequant_identical():
    """The conversion takes no nibble argument; a layer's nibble tensor is
    bit-identical before and after converting its scales."""
    wl = synth.WORKLOADS["tiny"]
    from block_quantized_expert_mxfp4_b200 import workload
    p = workload.mx_proj(0, 0, 0, wl.E, wl.I, wl.H, wl.code_lo, wl.code_hi)
    before = p.q.clone()
    nv = workload.to_nvfp4(p)
    torch.cuda.synchronize()
    assert torch.equal(before, nv.q) and nv.q.data_ptr() == p.q.data_ptr()
