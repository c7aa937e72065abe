"""Independent dequantization used only to pin the oracle in tests.

Built from library decoders (ml_dtypes' float4_e2m1fn / float8_e8m0fnu /
float8_e4m3fn) and numpy array operations, not from the oracle's code.  It
serves as the "second formulation" the oracle is checked against: decode the
whole matrix, then a library matmul.
"""
import ml_dtypes
import numpy as np

E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
E8M0 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def unpack_nibbles(q):
    """[..., K/2] bytes -> [..., K] codes; element 2i = low nibble of byte i."""
    q = np.asarray(q, dtype=np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = q & 0x0F
    out[..., 1::2] = q >> 4
    return out


def dequant_mx(q, s):
    """MXFP4 -> float64 [.., N, K]: e2m1 * 2^(c-127) per 32-block (np.repeat on K);
    exact (2 significant bits times a power of two)."""
    codes = unpack_nibbles(q)
    scale = np.repeat(E8M0[np.asarray(s)], 32, axis=-1)
    return E2M1[codes] * scale


def dequant_nv(q, s, s2):
    """NVFP4 -> float64: e2m1 * e4m3 per 16-block * per-expert fp32 scale_2;
    exact (at most 2 + 4 + 24 significant bits)."""
    codes = unpack_nibbles(q)
    scale = np.repeat(E4M3[np.asarray(s)], 16, axis=-1)
    s2 = np.asarray(s2, dtype=np.float32).astype(np.float64)
    s2 = s2.reshape((-1,) + (1,) * (codes.ndim - 1))
    return E2M1[codes] * scale * s2


def dequant_fp8(w, s, block=128):
    N, K = w.shape
    scale = np.kron(E8M0[np.asarray(s)], np.ones((block, block)))[:N, :K]
    return E4M3[np.asarray(w)] * scale


def bf16_to_f64(x):
    """bf16 bits (uint16 or int16 array, or a torch bf16 tensor) -> float64."""
    if hasattr(x, "float"):
        return x.float().double().numpy()
    u = np.asarray(x).view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
