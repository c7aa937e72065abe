"""ctypes binding of libqk.so: the C ABI of include/qk.h, same names.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); the stream defaults to torch's current stream.  If libqk.so is
missing or cannot be loaded, importing the functions raises -- there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqk.so")

QK_OK, QK_ERR_INVALID_ARG, QK_ERR_UNSUPPORTED, QK_ERR_WORKSPACE = 0, 1, 2, 3
QK_ERR_NAN_SCALE, QK_ERR_CUDA, QK_ERR_TIMEOUT, QK_ERR_NONFINITE = 4, 5, 6, 7
QK_FMT_MXFP4, QK_FMT_NVFP4 = 1, 2
QK_ACT_NONE, QK_ACT_MXFP4, QK_ACT_E4M3 = 0, 1, 2

# exported symbols (kept in sync with include/qk.h; checked by tests/test_abi.py)
SYMBOLS = (
    "moe_expert_workspace_size", "moe_expert_forward", "moe_route_topk",
    "quant_convert_mxfp4_to_nvfp4", "quant_convert_nvfp4_to_mxfp4", "fp8_block_linear",
    "fp8_shared_expert_workspace_size",
    "fp8_shared_expert_forward", "qk_last_device_status", "qk_status_string",
    "qk_debug_set_wait_limit_ns", "moe_expert_forward_noalloc",
)


class QkError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class qk_weight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("q", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("scale_2", ctypes.c_void_p), ("n_experts", ctypes.c_int32),
                ("rows", ctypes.c_int32), ("cols", ctypes.c_int32)]


class qk_moe_layer(ctypes.Structure):
    _fields_ = [("gate", qk_weight), ("up", qk_weight), ("down", qk_weight),
                ("hidden", ctypes.c_int32), ("inter", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libqk.so (built by ``python -m block_quantized_expert_mxfp4_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqk.so not built at {LIB_PATH}; run the package's build step")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    L.moe_expert_workspace_size.restype = sz
    L.moe_expert_workspace_size.argtypes = [ctypes.POINTER(qk_moe_layer), i32, i32, i32]
    L.moe_expert_forward.restype = i32
    L.moe_expert_forward.argtypes = [ctypes.POINTER(qk_moe_layer), vp, i32, vp, vp, i32, vp, i32,
                                     i32, vp, sz, vp]
    L.moe_expert_forward_noalloc.restype = i32
    L.moe_expert_forward_noalloc.argtypes = [ctypes.POINTER(qk_moe_layer), vp, i32, vp, vp, i32, vp,
                                             i32, vp]
    L.moe_route_topk.restype = i32
    L.moe_route_topk.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.quant_convert_mxfp4_to_nvfp4.restype = i32
    L.quant_convert_mxfp4_to_nvfp4.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
    L.quant_convert_nvfp4_to_mxfp4.restype = i32
    L.quant_convert_nvfp4_to_mxfp4.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
    L.fp8_block_linear.restype = i32
    L.fp8_block_linear.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp, i32, vp]
    L.fp8_shared_expert_workspace_size.restype = sz
    L.fp8_shared_expert_workspace_size.argtypes = [i32, i32, i32]
    L.fp8_shared_expert_forward.restype = i32
    L.fp8_shared_expert_forward.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz,
                                            vp]
    L.qk_last_device_status.restype = i32
    L.qk_last_device_status.argtypes = [vp]
    L.qk_status_string.restype = ctypes.c_char_p
    L.qk_status_string.argtypes = [i32]
    L.qk_debug_set_wait_limit_ns.restype = i32
    L.qk_debug_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, what: str):
    if rc != QK_OK:
        raise QkError(rc, what)


def status_string(code: int) -> str:
    return load().qk_status_string(code).decode()


def make_weight(fmt: int, q: torch.Tensor, scales: torch.Tensor,
                scale_2: Optional[torch.Tensor] = None) -> qk_weight:
    E, N, Kh = q.shape
    return qk_weight(fmt, q.data_ptr(), scales.data_ptr(),
                     None if scale_2 is None else scale_2.data_ptr(), E, N, 2 * Kh)


def make_layer(gate: qk_weight, up: qk_weight, down: qk_weight) -> qk_moe_layer:
    return qk_moe_layer(gate, up, down, gate.cols, gate.rows)


def moe_expert_workspace_size(layer: qk_moe_layer, n_tokens: int, top_k: int,
                              act_quant: int = QK_ACT_NONE) -> int:
    return load().moe_expert_workspace_size(ctypes.byref(layer), n_tokens, top_k, act_quant)


def moe_expert_forward(layer: qk_moe_layer, x: torch.Tensor, topk_ids: torch.Tensor,
                       topk_w: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                       act_quant: int = QK_ACT_NONE, stream=None) -> None:
    T = x.shape[0]
    k = topk_ids.shape[1] if topk_ids.dim() == 2 else 1
    rc = load().moe_expert_forward(ctypes.byref(layer), _ptr(x), T, _ptr(topk_ids), _ptr(topk_w),
                                   k, _ptr(y), int(y.dtype == torch.bfloat16), act_quant,
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc, "moe_expert_forward")


def moe_expert_forward_noalloc(layer: qk_moe_layer, x: torch.Tensor, topk_ids: torch.Tensor,
                               topk_w: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """moe_expert_forward with the library's fixed scratch array (no workspace)."""
    T = x.shape[0]
    k = topk_ids.shape[1] if topk_ids.dim() == 2 else 1
    rc = load().moe_expert_forward_noalloc(ctypes.byref(layer), _ptr(x), T, _ptr(topk_ids),
                                           _ptr(topk_w), k, _ptr(y), int(y.dtype == torch.bfloat16),
                                           _stream(stream))
    _check(rc, "moe_expert_forward_noalloc")


def moe_route_topk(logits: torch.Tensor, top_k: int, ids: torch.Tensor, w: torch.Tensor,
                   stream=None) -> None:
    T, E = logits.shape
    _check(load().moe_route_topk(_ptr(logits), T, E, top_k, _ptr(ids), _ptr(w), _stream(stream)),
           "moe_route_topk")


def quant_convert_mxfp4_to_nvfp4(e8m0: torch.Tensor, e4m3: torch.Tensor, scale_2: torch.Tensor,
                                 n_inexact: torch.Tensor, stream=None) -> None:
    E, N, K32 = e8m0.shape
    _check(load().quant_convert_mxfp4_to_nvfp4(_ptr(e8m0), E, N, 32 * K32, _ptr(e4m3),
                                               _ptr(scale_2), _ptr(n_inexact), _stream(stream)),
           "quant_convert_mxfp4_to_nvfp4")


def quant_convert_nvfp4_to_mxfp4(e4m3: torch.Tensor, scale_2: torch.Tensor, e8m0: torch.Tensor,
                                 n_inexact: torch.Tensor, stream=None) -> None:
    E, N, K16 = e4m3.shape
    _check(load().quant_convert_nvfp4_to_mxfp4(_ptr(e4m3), _ptr(scale_2), E, N, 16 * K16, _ptr(e8m0),
                                               _ptr(n_inexact), _stream(stream)),
           "quant_convert_nvfp4_to_mxfp4")


def fp8_block_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor, y: torch.Tensor,
                     stream=None, scale_block: int = 128) -> None:
    M, K = x.shape
    N = w.shape[0]
    _check(load().fp8_block_linear(_ptr(x), M, K, _ptr(w), _ptr(w_scale), N, scale_block, _ptr(y),
                                   int(y.dtype == torch.bfloat16), _stream(stream)),
           "fp8_block_linear")


def fp8_shared_expert_workspace_size(M: int, hidden: int, inter: int) -> int:
    return load().fp8_shared_expert_workspace_size(M, hidden, inter)


def fp8_shared_expert_forward(x, wg, sg, wu, su, wd, sd, y, workspace, stream=None,
                              scale_block: int = 128) -> None:
    M, H = x.shape
    I = wg.shape[0]
    _check(load().fp8_shared_expert_forward(
        _ptr(x), M, H, I, _ptr(wg), _ptr(sg), _ptr(wu), _ptr(su), _ptr(wd), _ptr(sd), scale_block,
        _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "fp8_shared_expert_forward")


def qk_last_device_status(stream=None) -> int:
    return load().qk_last_device_status(_stream(stream))


def qk_debug_set_wait_limit_ns(limit_ns: int) -> None:
    _check(load().qk_debug_set_wait_limit_ns(limit_ns), "qk_debug_set_wait_limit_ns")
