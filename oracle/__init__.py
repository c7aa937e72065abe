"""CPU oracle for the block-quantized expert FFN -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It loads ``liboracle.so`` built from
``qk_oracle.c`` (plain C99, fp64 accumulation) and shares no code with the CUDA
library.  See ``qk_oracle.h`` for the definitions it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")

QKO_OK, QKO_ERR_INVALID_ARG, QKO_ERR_NAN_SCALE = 0, 1, 4
MXFP4, NVFP4 = 1, 2
ACT_NONE, ACT_MXFP4, ACT_E4M3 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (C99, -O2, no FP contraction, OpenMP)."""
    src = os.path.join(_HERE, "qk_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "qk_oracle.h"))):
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", src, "-o", _SO, "-lm"]
        subprocess.check_call(cmd)
    return _SO


class _Weight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("q", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("scale_2", ctypes.c_void_p), ("n_experts", ctypes.c_int32),
                ("rows", ctypes.c_int32), ("cols", ctypes.c_int32)]


class _Layer(ctypes.Structure):
    _fields_ = [("gate", _Weight), ("up", _Weight), ("down", _Weight),
                ("hidden", ctypes.c_int32), ("inter", ctypes.c_int32)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
        L.qko_e2m1_value.restype = f64
        L.qko_e2m1_value.argtypes = [ctypes.c_uint8]
        L.qko_e8m0_value.restype = f64
        L.qko_e8m0_value.argtypes = [ctypes.c_uint8]
        L.qko_e4m3_value.restype = f64
        L.qko_e4m3_value.argtypes = [ctypes.c_uint8]
        L.qko_e4m3_encode.restype = ctypes.c_uint8
        L.qko_e4m3_encode.argtypes = [f64]
        L.qko_e2m1_encode.restype = ctypes.c_uint8
        L.qko_e2m1_encode.argtypes = [f64]
        L.qko_act_quant.argtypes = [vp, i32, i32, vp, vp, vp]
        L.qko_moe_forward_aq.argtypes = [ctypes.POINTER(_Layer), vp, i32, vp, vp, i32, i32, vp]
        L.qko_expert_ffn_aq.argtypes = [ctypes.POINTER(_Layer), i32, vp, i32, vp, vp, vp, vp]
        L.qko_dequant_row.argtypes = [ctypes.POINTER(_Weight), i32, i32, vp]
        L.qko_convert_mx_to_nv.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.qko_convert_nv_to_mx.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        L.qko_route_topk.argtypes = [vp, i32, i32, i32, vp, vp]
        L.qko_moe_forward.argtypes = [ctypes.POINTER(_Layer), vp, i32, vp, vp, i32, vp]
        L.qko_expert_ffn.argtypes = [ctypes.POINTER(_Layer), i32, vp, vp, vp, vp, vp]
        L.qko_fp8_block_linear.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp]
        L.qko_fp8_swiglu_ffn.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp]
        L.qko_set_threads.argtypes = [i32]
        L.qko_get_threads.restype = i32
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle status {code}")
        self.code = code


def _chk(rc):
    if rc != QKO_OK:
        raise OracleError(rc)


def _np(a, dtype):
    """Contiguous numpy view of a CPU torch tensor or numpy array."""
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if a.dtype.__str__() == "torch.bfloat16":
            a = a.view(__import__("torch").int16)
        a = a.numpy()
    return np.ascontiguousarray(a).view(dtype) if a.dtype != dtype else np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().qko_set_threads(n)


def get_threads() -> int:
    return lib().qko_get_threads()


def e2m1_value(code: int) -> float:
    return lib().qko_e2m1_value(code)


def e8m0_value(code: int) -> float:
    return lib().qko_e8m0_value(code)


def e4m3_value(code: int) -> float:
    return lib().qko_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return lib().qko_e4m3_encode(float(v))


class Weight:
    """One projection in the storage layout (CPU arrays kept alive here)."""

    def __init__(self, fmt, q, scales, scale_2=None):
        self.fmt = fmt
        self.q = _np(q, np.uint8)
        self.scales = _np(scales, np.uint8)
        self.scale_2 = None if scale_2 is None else _np(scale_2, np.float32)
        E, N, Kh = self.q.shape
        self.E, self.N, self.K = E, N, 2 * Kh

    def c(self):
        return _Weight(self.fmt, self.q.ctypes.data, self.scales.ctypes.data,
                       None if self.scale_2 is None else self.scale_2.ctypes.data,
                       self.E, self.N, self.K)


class Layer:
    def __init__(self, gate: Weight, up: Weight, down: Weight):
        self.gate, self.up, self.down = gate, up, down
        self.hidden, self.inter = gate.K, gate.N

    def c(self):
        return _Layer(self.gate.c(), self.up.c(), self.down.c(), self.hidden, self.inter)


def dequant(w: Weight, e: int) -> np.ndarray:
    """Expert e's dequantized matrix [N][K], exact (float64)."""
    out = np.empty((w.N, w.K), dtype=np.float64)
    cw = w.c()
    for n in range(w.N):
        _chk(lib().qko_dequant_row(ctypes.byref(cw), e, n, _p(out[n])))
    return out


def convert_mx_to_nv(e8m0) -> tuple:
    """Returns (e4m3 [E][N][K/16] uint8, scale_2 [E] float32, n_inexact)."""
    s = _np(e8m0, np.uint8)
    E, N, K32 = s.shape
    out = np.empty((E, N, 2 * K32), dtype=np.uint8)
    s2 = np.empty(E, dtype=np.float32)
    n_bad = ctypes.c_uint64(0)
    _chk(lib().qko_convert_mx_to_nv(_p(s), E, N, 32 * K32, _p(out), _p(s2), ctypes.byref(n_bad)))
    return out, s2, int(n_bad.value)


def convert_nv_to_mx(e4m3, scale_2) -> tuple:
    """e4m3 [E][N][K/16] + scale_2 [E] -> (e8m0 [E][N][K/32] uint8, n_inexact)."""
    s = _np(e4m3, np.uint8)
    s2 = np.ascontiguousarray(_np(scale_2, np.float32).reshape(-1))
    E, N, K16 = s.shape
    out = np.empty((E, N, K16 // 2), dtype=np.uint8)
    n_bad = ctypes.c_uint64(0)
    _chk(lib().qko_convert_nv_to_mx(_p(s), _p(s2), E, N, 16 * K16, _p(out), ctypes.byref(n_bad)))
    return out, int(n_bad.value)


def route_topk(logits, k: int):
    lg = _np(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _chk(lib().qko_route_topk(_p(lg), T, E, k, _p(ids), _p(w)))
    return ids, w


def moe_forward(layer: Layer, x_bf16, ids, w, aq: int = ACT_NONE) -> np.ndarray:
    x = _np(x_bf16, np.uint16)
    ids = _np(ids, np.int32)
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float64))
    T, k = ids.shape
    y = np.empty((T, layer.hidden), dtype=np.float64)
    cl = layer.c()
    _chk(lib().qko_moe_forward_aq(ctypes.byref(cl), _p(x), T, _p(ids), _p(w), k, aq, _p(y)))
    return y


def expert_ffn(layer: Layer, e: int, x_bf16_row, aq: int = ACT_NONE):
    """(g, u, h, d) of expert e on one token; with `aq`, h is the quantized
    h that the down projection consumes."""
    x = _np(x_bf16_row, np.uint16).reshape(-1)
    I, H = layer.inter, layer.hidden
    g, u, h = (np.empty(I) for _ in range(3))
    d = np.empty(H)
    cl = layer.c()
    _chk(lib().qko_expert_ffn_aq(ctypes.byref(cl), e, _p(x), aq, _p(g), _p(u), _p(h), _p(d)))
    return g, u, h, d


def e2m1_encode(v: float) -> int:
    return lib().qko_e2m1_encode(float(v))


def act_quant(v, aq: int):
    """Quantize a float64 vector (length a multiple of 32) by the OCP MX rule:
    returns (element codes uint8 [n], e8m0 scale codes uint8 [n/32],
    dequantized float64 [n])."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64).reshape(-1))
    codes = np.empty(v.size, np.uint8)
    scales = np.empty(v.size // 32, np.uint8)
    out = np.empty(v.size, np.float64)
    _chk(lib().qko_act_quant(_p(v), v.size, aq, _p(codes), _p(scales), _p(out)))
    return codes, scales, out


def fp8_block_linear(x_bf16, w, w_scale, block: int = 128) -> np.ndarray:
    x = _np(x_bf16, np.uint16)
    wq = _np(w, np.uint8)
    ws = _np(w_scale, np.uint8)
    M, K = x.shape
    N = wq.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _chk(lib().qko_fp8_block_linear(_p(x), M, K, _p(wq), _p(ws), N, block, _p(y)))
    return y


def fp8_swiglu_ffn(x_bf16, wg, sg, wu, su, wd, sd, block: int = 128) -> np.ndarray:
    x = _np(x_bf16, np.uint16)
    M, H = x.shape
    arrs = [_np(a, np.uint8) for a in (wg, sg, wu, su, wd, sd)]
    I = arrs[0].shape[0]
    y = np.empty((M, H), dtype=np.float64)
    _chk(lib().qko_fp8_swiglu_ffn(_p(x), M, H, I, *[_p(a) for a in arrs], block, _p(y)))
    return y
