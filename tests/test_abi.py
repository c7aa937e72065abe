"""The C-ABI library loads on a CPU-only host and exports every symbol the
header declares; host-side argument validation returns its status codes
without touching a GPU."""
import ctypes
import os
import re

import pytest

import block_quantized_expert_mxfp4_b200 as qk
from block_quantized_expert_mxfp4_b200 import _lib
from conftest import ROOT


def _declared():
    hdr = open(os.path.join(ROOT, "include", "qk.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_0-9]+)\s*\(", hdr, re.M)


def test_library_exports_every_declared_symbol():
    L = qk.load()
    names = _declared()
    assert len(names) == 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.SYMBOLS)


def test_status_strings():
    for code in range(8):
        assert qk.status_string(code) not in ("", "unknown status")
    assert qk.status_string(99) == "unknown status"


def _fake_layer(H=4096, I=2048, E=256, fmts=(1, 1, 1)):
    base = 1 << 20  # fake 16-aligned addresses: never dereferenced on these paths
    ws = []
    for i, ((r, c), f) in enumerate(zip(((I, H), (I, H), (H, I)), fmts)):
        ws.append(_lib.qk_weight(f, base * (3 * i + 1), base * (3 * i + 2),
                                 base * (3 * i + 3) if f == 2 else None, E, r, c))
    return _lib.make_layer(*ws)


def test_workspace_query_and_shape_validation():
    L = qk.load()
    lay = _fake_layer()
    n1 = L.moe_expert_workspace_size(ctypes.byref(lay), 1, 6, 0)
    n16 = L.moe_expert_workspace_size(ctypes.byref(lay), 16, 6, 0)
    assert 0 < n1 < n16
    assert L.moe_expert_workspace_size(ctypes.byref(lay), 1, 9, 0) == 0        # top_k > 8
    assert L.moe_expert_workspace_size(ctypes.byref(_fake_layer(H=4096 + 64)), 1, 6, 0) == 0
    assert L.moe_expert_workspace_size(ctypes.byref(_fake_layer(fmts=(1, 3, 1))), 1, 6, 0) == 0
    bad = _fake_layer()
    bad.down.rows = 2048
    assert L.moe_expert_workspace_size(ctypes.byref(bad), 1, 6, 0) == 0
    nv = _fake_layer(fmts=(2, 2, 2))
    nv.up.scale_2 = None
    assert L.moe_expert_workspace_size(ctypes.byref(nv), 1, 6, 0) == 0


def test_workspace_query_follows_the_path_choice():
    """All-MXFP4 layers with 32-byte aligned weights take the block-scaled
    decode and grouped paths (their own workspace layouts); the same layer
    with misaligned weights, or in NVFP4, takes the f16 paths, whose
    workspace depends on the shapes only."""
    L = qk.load()
    mx = _fake_layer()
    nv = _fake_layer(fmts=(2, 2, 2))
    mis = _fake_layer()
    mis.gate.q = mis.gate.q + 16  # 16-byte aligned, not 32: no block-scaled path
    for T in (1, 16, 100):         # decode (<= 21 tokens at top-6) and grouped
        a, b, c = (L.moe_expert_workspace_size(ctypes.byref(x), T, 6, 0) for x in (mx, nv, mis))
        assert a > 0 and b > 0
        assert c == b and a != b, (T, a, b, c)


def test_workspace_query_with_activation_modes():
    """The quantized modes run the grouped block-scaled kernels at every token
    count: their workspace is the grouped one (the bf16 query's size above one
    decode launch), and 0 where the mode is refused.  An all-NVFP4 layer runs
    QK_ACT_MXFP4 on kind::mxf4nvf4 (twice the token scale atoms and two
    per-row factor arrays beyond the MXFP4 layout); W4A8 has no NVFP4 form."""
    L = qk.load()
    q = lambda lay, T, aq: L.moe_expert_workspace_size(ctypes.byref(lay), T, 6, aq)
    mx, nv, mis = _fake_layer(), _fake_layer(fmts=(2, 2, 2)), _fake_layer()
    mis.gate.q = mis.gate.q + 16
    mixed = _fake_layer(fmts=(1, 2, 1))
    for aq in (qk.QK_ACT_MXFP4, qk.QK_ACT_E4M3):
        assert q(mx, 100, aq) == q(mx, 100, qk.QK_ACT_NONE) > 0
        assert q(mx, 1, aq) > 0 and q(mx, 1, aq) != q(mx, 1, qk.QK_ACT_NONE)
        assert q(mx, 1, aq) < q(mx, 16, aq) < q(mx, 100, aq)
        assert q(mis, 1, aq) == 0 and q(mixed, 1, aq) == 0
    assert q(nv, 1, qk.QK_ACT_E4M3) == 0
    for T in (1, 16, 100):
        assert q(nv, T, qk.QK_ACT_MXFP4) > q(mx, T, qk.QK_ACT_MXFP4)
    nvmis = _fake_layer(fmts=(2, 2, 2))
    nvmis.down.scales = nvmis.down.scales + 8
    assert q(nvmis, 1, qk.QK_ACT_MXFP4) == 0
    assert q(mx, 1, 7) == 0


def test_noalloc_limit_in_pairs():
    """16 MiB of fixed scratch: at hidden 4096, inter 2048 the block-scaled
    MXFP4 decode needs about 96 KiB per pair, so every decode launch (up to
    128 pairs) fits, while the grouped kernels above 128 pairs do not; the
    f16 decode for NVFP4 layers fits 114 pairs at top-6 and 118 at top-2."""
    L = qk.load()
    mx, nv = _fake_layer(), _fake_layer(fmts=(2, 2, 2))
    cap = 16 << 20
    q = lambda lay, T, k: L.moe_expert_workspace_size(ctypes.byref(lay), T, k, 0)
    assert q(mx, 21, 6) <= cap < q(mx, 22, 6)      # 126 pairs (decode) fit, 132 (grouped) do not
    assert q(mx, 64, 2) <= cap < q(mx, 65, 2)      # 128 / 130
    assert q(nv, 19, 6) <= cap < q(nv, 20, 6)      # 114 / 120
    assert q(nv, 59, 2) <= cap < q(nv, 60, 2)      # 118 / 120


def test_forward_argument_errors_are_synchronous():
    L = qk.load()
    lay = _fake_layer()
    vp = ctypes.c_void_p
    f = L.moe_expert_forward
    p = vp(1 << 24)
    ws = L.moe_expert_workspace_size(ctypes.byref(lay), 1, 6, 0)
    assert f(ctypes.byref(lay), p, 0, p, p, 6, p, 0, 0, p, ws, None) == qk.QK_OK  # T = 0
    assert f(ctypes.byref(lay), p, 1, p, p, 6, p, 0, 7, p, ws, None) == qk.QK_ERR_INVALID_ARG  # mode
    nv = _fake_layer(fmts=(2, 2, 2))
    for aq in (qk.QK_ACT_MXFP4, qk.QK_ACT_E4M3):
        # a quantized mode: an all-MXFP4 layer runs the grouped kernels, whose
        # workspace the bf16-path size does not cover; NVFP4 layers likewise in
        # QK_ACT_MXFP4, and are refused in QK_ACT_E4M3
        assert f(ctypes.byref(lay), p, 1, p, p, 6, p, 0, aq, p, ws, None) == qk.QK_ERR_WORKSPACE
        want = qk.QK_ERR_WORKSPACE if aq == qk.QK_ACT_MXFP4 else qk.QK_ERR_UNSUPPORTED
        assert f(ctypes.byref(nv), p, 1, p, p, 6, p, 0, aq, p, 1024, None) == want
    assert f(ctypes.byref(lay), p, 1, p, p, 6, p, 0, 0, p, ws - 1, None) == qk.QK_ERR_WORKSPACE
    assert f(ctypes.byref(lay), p, 1, p, p, 6, p, 0, 0, None, ws, None) == qk.QK_ERR_WORKSPACE
    assert f(ctypes.byref(lay), None, 1, p, p, 6, p, 0, 0, p, ws, None) == qk.QK_ERR_INVALID_ARG
    assert f(ctypes.byref(lay), vp((1 << 24) + 8), 1, p, p, 6, p, 0, 0, p, ws, None) == \
        qk.QK_ERR_INVALID_ARG                                               # x not 16-B aligned
    assert f(None, p, 1, p, p, 6, p, 0, 0, p, ws, None) == qk.QK_ERR_INVALID_ARG
    assert L.moe_route_topk(p, 4, 8, 9, p, p, None) == qk.QK_ERR_INVALID_ARG  # k > E
    assert L.moe_route_topk(p, 0, 8, 2, p, p, None) == qk.QK_OK
    assert L.quant_convert_mxfp4_to_nvfp4(p, 2, 4, 48, p, p, p, None) == qk.QK_ERR_INVALID_ARG
    assert L.quant_convert_nvfp4_to_mxfp4(p, p, 2, 4, 48, p, p, None) == qk.QK_ERR_INVALID_ARG
    assert L.quant_convert_nvfp4_to_mxfp4(None, p, 2, 4, 64, p, p, None) == qk.QK_ERR_INVALID_ARG
    assert L.fp8_block_linear(p, 1, 100, p, p, 16, 128, p, 0, None) == qk.QK_ERR_INVALID_ARG
    assert L.fp8_block_linear(p, 1, 128, p, p, 16, 64, p, 0, None) == qk.QK_ERR_INVALID_ARG  # tile
    assert L.fp8_shared_expert_workspace_size(8, 4096, 2048) > 0
    assert L.fp8_shared_expert_forward(p, 8, 4096, 2048, p, p, p, p, p, p, 128, p, p, 0, None) == \
        qk.QK_ERR_WORKSPACE
    assert L.fp8_shared_expert_forward(p, 8, 4096, 2048, p, p, p, p, p, p, 16, p, p, 1 << 30, None) == \
        qk.QK_ERR_INVALID_ARG


def test_noalloc_entry_rejects_before_any_device_work():
    L = qk.load()
    lay = _fake_layer()
    p = ctypes.c_void_p(1 << 24)
    f = L.moe_expert_forward_noalloc
    assert f(ctypes.byref(lay), p, 0, p, p, 6, p, 0, None) == qk.QK_OK                # T = 0
    assert f(ctypes.byref(lay), p, 22, p, p, 6, p, 0, None) == qk.QK_ERR_WORKSPACE    # > 16 MiB (grouped)
    assert f(ctypes.byref(lay), p, 1, p, p, 9, p, 0, None) == qk.QK_ERR_INVALID_ARG   # top_k > 8
    assert f(None, p, 1, p, p, 6, p, 0, None) == qk.QK_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_wrappers_of_the_newer_arguments_marshal_them():
    """The Python wrappers pass scale_block, act_quant and the reverse
    conversion's arguments in the header's order: each invalid value comes
    back as its synchronous error (stream 0: no device is touched)."""
    import torch

    def code(fn):
        with pytest.raises(qk.QkError) as ei:
            fn()
        return ei.value.code

    e4 = torch.zeros((2, 4, 3), dtype=torch.uint8)             # K = 48: not a multiple of 32
    assert code(lambda: qk.quant_convert_nvfp4_to_mxfp4(e4, torch.ones(2), torch.zeros((2, 4, 1), dtype=torch.uint8),
                                                        torch.zeros(1, dtype=torch.int64), stream=0)) == \
        qk.QK_ERR_INVALID_ARG
    x = torch.zeros((1, 128), dtype=torch.bfloat16)
    w = torch.zeros((16, 128), dtype=torch.uint8)
    s = torch.zeros((1, 4), dtype=torch.uint8)
    y = torch.zeros((1, 16))
    assert code(lambda: qk.fp8_block_linear(x, w, s, y, stream=0, scale_block=64)) == qk.QK_ERR_INVALID_ARG
    wg = torch.zeros((128, 128), dtype=torch.uint8)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    assert code(lambda: qk.fp8_shared_expert_forward(x, wg, s, wg, s, wg, s, torch.zeros((1, 128)), ws,
                                                     stream=0, scale_block=16)) == qk.QK_ERR_INVALID_ARG
    lay = _fake_layer()
    ids = torch.zeros((1, 6), dtype=torch.int32)
    wt = torch.zeros((1, 6))
    yy = torch.zeros((1, 4096))
    assert code(lambda: qk.moe_expert_forward(lay, torch.zeros((1, 4096), dtype=torch.bfloat16), ids, wt, yy, ws,
                                              act_quant=7, stream=0)) == qk.QK_ERR_INVALID_ARG
    assert qk.moe_expert_workspace_size(lay, 1, 6, 7) == 0
    assert qk.moe_expert_workspace_size(lay, 1, 6, qk.QK_ACT_E4M3) > 0
