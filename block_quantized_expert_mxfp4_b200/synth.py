"""Seeded synthetic inputs for the block-quantized expert FFN.

This module only *draws* inputs: random weight bytes, random scale codes,
normal activations and router logits, and Zipf-skewed expert choices.  It holds
none of the method's arithmetic (no decoding, no dot products, no softmax, no
conversion), so both the CUDA path and the CPU oracle may take their inputs
from it.

Weight bytes come from a counter-based generator so that any slice (one expert
of one projection of one layer) can be regenerated on the host without
materialising the rest.  The generator is SplitMix64 (Steele, Lea, Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014), the output
function applied to ``key + i`` for element/word ``i``.  It is implemented
twice: with numpy ``uint64`` on the host and with torch ``int64`` on any device
(torch wraps signed 64-bit products; right shifts are masked to make them
logical).  ``tests/test_synth.py`` checks the two give the same bytes.

Activations and logits are drawn on the host with numpy's PCG64 and uploaded.

Workload recipes (shapes from the DeepSeek-V4-Flash base-model table: hidden
4096, 256 routed experts, top-6, 43 layers; REAP-K180 page: 180 experts per
layer; expert intermediate 2048):

* ``tiny``       E=8,   k=2, H=256,  I=128,  T=4,    MXFP4, e8m0 codes 121..129
* ``decode_mx``  E=256, k=6, H=4096, I=2048, T=1,    MXFP4, e8m0 codes 118..127
* ``decode_nv``  same weights converted to NVFP4, T in {1, 4, 16}
* ``prefill``    E=256, k=6, H=4096, I=2048, T=2048, MXFP4, Zipf(s=1) routing
* ``stack43``    43 layers, E=180, k=6, T=8, per-(layer, projection) MXFP4 or
  NVFP4, plus an FP8 E4M3 block-128 shared expert 4096x2048.

General NVFP4 sources (not converted from MXFP4): the same nibble bytes, e4m3
block-scale codes uniform in ``[NV_CODE_LO, NV_CODE_HI]`` (32 .. 448, every
mantissa) and a per-expert fp32 ``scale_2`` in [2^-13, 2^-12) with a full
24-bit significand, so neither scale is a power of two in general.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = [
    "WORKLOADS", "Workload", "splitmix64_np", "splitmix64_torch", "tensor_key",
    "random_bytes", "scale_codes", "fp8_codes", "activations", "router_logits",
    "zipf_logits", "format_choice", "TID", "NV_CODE_LO", "NV_CODE_HI", "nv_scale_2",
    "nv_expert_bytes", "mx_expert_bytes",
]

_C0 = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_M64 = (1 << 64) - 1


def _to_i64(v: int) -> int:
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


def splitmix64_int(x: int) -> int:
    """SplitMix64 output function on a Python int (reference for the others)."""
    z = (x + _C0) & _M64
    z = ((z ^ (z >> 30)) * _C1) & _M64
    z = ((z ^ (z >> 27)) * _C2) & _M64
    return z ^ (z >> 31)


def splitmix64_np(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a numpy uint64 array (wrapping arithmetic)."""
    x = x.astype(np.uint64, copy=False)
    with np.errstate(over="ignore"):
        z = x + np.uint64(_C0)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_C1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_C2)
        return z ^ (z >> np.uint64(31))


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64_torch(x: torch.Tensor) -> torch.Tensor:
    """SplitMix64 output function on a torch int64 tensor (bit pattern = uint64)."""
    z = x + _to_i64(_C0)
    z = (z ^ _lsr(z, 30)) * _to_i64(_C1)
    z = (z ^ _lsr(z, 27)) * _to_i64(_C2)
    return z ^ _lsr(z, 31)


def tensor_key(seed: int, tid: int) -> int:
    """64-bit stream key of tensor ``tid`` under ``seed``."""
    return splitmix64_int((seed * 0x100000001B3) ^ splitmix64_int(tid))


class TID:
    """Tensor ids: one independent stream per (layer, projection, kind)."""

    GATE, UP, DOWN, SH_GATE, SH_UP, SH_DOWN = range(6)
    NIBBLES, SCALES, NV_SCALES, NV_SCALE_2 = 0, 1, 2, 3

    @staticmethod
    def of(layer: int, proj: int, kind: int) -> int:
        return (layer << 8) | (proj << 4) | kind


_CHUNK = 1 << 24  # hashes per torch chunk (bounded temporaries)


def _hash_words(key: int, start: int, n: int, device) -> torch.Tensor:
    """int64 tensor of SplitMix64(key + start + i) for i < n on ``device``."""
    dev = torch.device(device)
    if dev.type == "cpu":
        idx = np.arange(start, start + n, dtype=np.uint64) + np.uint64(key)
        return torch.from_numpy(splitmix64_np(idx).view(np.int64))
    out = torch.empty(n, dtype=torch.int64, device=dev)
    base = _to_i64(key + start)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        idx = torch.arange(c0, c1, dtype=torch.int64, device=dev) + base
        out[c0:c1] = splitmix64_torch(idx)
    return out


def random_bytes(seed: int, tid: int, n: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """``n`` uniform bytes of stream ``tid``, starting at byte ``offset``.

    Byte ``j`` of the stream is byte ``j % 8`` (little-endian) of word ``j // 8``.
    ``offset`` must be a multiple of 8 so a slice starts on a word.
    """
    assert offset % 8 == 0
    nw = (n + 7) // 8
    w = _hash_words(tensor_key(seed, tid), offset // 8, nw, device)
    return w.view(torch.uint8)[:n].clone() if (nw * 8 != n) else w.view(torch.uint8)


def scale_codes(seed: int, tid: int, n: int, lo: int, hi: int, device="cpu",
                offset: int = 0) -> torch.Tensor:
    """``n`` 8-bit codes uniform in ``[lo, hi]``: code j = lo + (w_j>>32)*(hi-lo+1)>>32."""
    span = hi - lo + 1
    w = _hash_words(tensor_key(seed, tid), offset, n, device)
    r = ((_lsr(w, 32) * span) >> 32) + lo
    return r.to(torch.uint8)


def fp8_codes(seed: int, tid: int, n: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """``n`` E4M3FN codes uniform over the 254 non-NaN codes (0x7F, 0xFF skipped)."""
    r = scale_codes(seed, tid, n, 0, 253, device, offset).to(torch.int32)
    r = torch.where(r >= 127, r + 1, r)
    return r.to(torch.uint8)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def activations(seed: int, T: int, H: int, stream: int = 1) -> torch.Tensor:
    """bf16 [T][H] with N(0,1) values (drawn in fp32, rounded to bf16 by torch)."""
    x = _rng(seed, 1000 + stream).standard_normal((T, H), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def router_logits(seed: int, T: int, E: int, stream: int = 1) -> torch.Tensor:
    """fp32 [T][E] router logits, N(0,1)."""
    return torch.from_numpy(_rng(seed, 2000 + stream).standard_normal((T, E), dtype=np.float32))


def zipf_logits(seed: int, T: int, E: int, k: int, s: float = 1.0, stream: int = 1) -> torch.Tensor:
    """Router logits that select a Zipf-skewed set of ``k`` experts per token.

    Expert popularity ranks are a seeded permutation of the experts with
    p(rank r) proportional to r**-s.  Each token's ``k`` experts are drawn
    without replacement in proportion to p (Gumbel-top-k: the ``k`` largest
    ``log p + Gumbel`` keys).  The chosen experts get fresh N(0,1) logits and
    all others ``-inf``, so softmax-top-k routing over these logits returns
    exactly the chosen set, with combine weights a softmax of the ``k`` fresh
    logits.
    """
    rng = _rng(seed, 3000 + stream)
    perm = rng.permutation(E)
    logp = np.empty(E, dtype=np.float64)
    logp[perm] = -s * np.log(np.arange(1, E + 1, dtype=np.float64))
    g = rng.gumbel(size=(T, E))
    keys = logp[None, :] + g
    chosen = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    out = np.full((T, E), -np.inf, dtype=np.float32)
    vals = rng.standard_normal((T, k), dtype=np.float32)
    np.put_along_axis(out, chosen, vals, axis=1)
    return torch.from_numpy(out)


def format_choice(seed: int, n_layers: int) -> np.ndarray:
    """Seeded per-(layer, projection) format: 1 = MXFP4, 2 = NVFP4; shape [L][3]."""
    return _rng(seed, 4000).integers(1, 3, size=(n_layers, 3)).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    E: int
    k: int
    H: int
    I: int
    T: int
    code_lo: int
    code_hi: int
    layers: int = 1
    fmt: str = "mx"          # "mx", "nv" or "mixed"
    routing: str = "softmax"  # "softmax" or "zipf"
    shared_fp8: bool = False


WORKLOADS = {
    "tiny": Workload("tiny", 8, 2, 256, 128, 4, 121, 129),
    "decode_mx": Workload("decode_mx", 256, 6, 4096, 2048, 1, 118, 127),
    "decode_nv": Workload("decode_nv", 256, 6, 4096, 2048, 1, 118, 127, fmt="nv"),
    "prefill": Workload("prefill", 256, 6, 4096, 2048, 2048, 118, 127, routing="zipf"),
    "stack43": Workload("stack43", 180, 6, 4096, 2048, 8, 118, 127, layers=43, fmt="mixed",
                        shared_fp8=True),
}


def mx_expert_bytes(seed: int, layer: int, proj: int, E_rows: int, K: int, lo: int, hi: int,
                    experts: Optional[Sequence[int]], n_experts: int, device="cpu"):
    """Nibble bytes [e][N][K/2] and e8m0 codes [e][N][K/32] of one projection.

    ``experts=None`` generates all ``n_experts``; otherwise only the listed ones
    (same bytes as the full tensor's slices).  ``E_rows`` is N, the rows per expert.
    """
    nb = E_rows * K // 2
    ns = E_rows * K // 32
    tq = TID.of(layer, proj, TID.NIBBLES)
    ts = TID.of(layer, proj, TID.SCALES)
    if experts is None:
        q = random_bytes(seed, tq, n_experts * nb, device).view(n_experts, E_rows, K // 2)
        s = scale_codes(seed, ts, n_experts * ns, lo, hi, device).view(n_experts, E_rows, K // 32)
        return q, s
    qs, ss = [], []
    for e in experts:
        qs.append(random_bytes(seed, tq, nb, device, offset=e * nb).view(E_rows, K // 2))
        ss.append(scale_codes(seed, ts, ns, lo, hi, device, offset=e * ns).view(E_rows, K // 32))
    return torch.stack(qs), torch.stack(ss)


NV_CODE_LO, NV_CODE_HI = 0x60, 0x7E  # e4m3 32 .. 448 (0x7F is NaN)


def nv_scale_2(seed: int, layer: int, proj: int, n_experts: int) -> np.ndarray:
    """fp32 ``scale_2`` [n_experts] of a general NVFP4 projection:
    (2^23 + m) * 2^-36 with m the top 23 bits of word e of the projection's
    stream, so every value lies in [2^-13, 2^-12) and is an exact fp32."""
    key = tensor_key(seed, TID.of(layer, proj, TID.NV_SCALE_2))
    w = _hash_words(key, 0, n_experts, "cpu").numpy().view(np.uint64)
    m = (w >> np.uint64(41)).astype(np.float64)
    return ((2.0 ** 23 + m) * 2.0 ** -36).astype(np.float32)


def nv_expert_bytes(seed: int, layer: int, proj: int, E_rows: int, K: int,
                    experts: Optional[Sequence[int]], n_experts: int, device="cpu",
                    code_lo: int = NV_CODE_LO, code_hi: int = NV_CODE_HI):
    """A general NVFP4 projection: nibble bytes [e][N][K/2] (the stream of the
    MXFP4 bytes), e4m3 block-scale codes [e][N][K/16] uniform in
    ``[code_lo, code_hi]`` and fp32 ``scale_2`` [e].

    ``experts=None`` generates all ``n_experts``; otherwise only the listed ones
    (same bytes as the full tensor's slices).
    """
    if not 0 <= code_lo <= code_hi <= 0x7E:
        raise ValueError("e4m3 block-scale codes must lie in [0, 0x7E] (0x7F is NaN)")
    nb = E_rows * K // 2
    ns = E_rows * K // 16
    tq = TID.of(layer, proj, TID.NIBBLES)
    ts = TID.of(layer, proj, TID.NV_SCALES)
    s2 = torch.from_numpy(nv_scale_2(seed, layer, proj, n_experts))
    if experts is None:
        q = random_bytes(seed, tq, n_experts * nb, device).view(n_experts, E_rows, K // 2)
        s = scale_codes(seed, ts, n_experts * ns, code_lo, code_hi, device).view(
            n_experts, E_rows, K // 16)
        return q, s, s2.to(device)
    qs, ss = [], []
    for e in experts:
        qs.append(random_bytes(seed, tq, nb, device, offset=e * nb).view(E_rows, K // 2))
        ss.append(scale_codes(seed, ts, ns, code_lo, code_hi, device, offset=e * ns).view(
            E_rows, K // 16))
    return torch.stack(qs), torch.stack(ss), s2[list(experts)].to(device)
