"""Device-resident synthetic workloads built from the seeded generators.

Weights are generated on the GPU by the counter-based generator in ``synth``
(the host can regenerate any expert's bytes independently); NVFP4 projections
are produced from MXFP4 ones by the library's own scale-only conversion, or,
for a general NVFP4 source, drawn directly (e4m3 block scales and scale_2 that
are not powers of two).  This module only allocates and fills tensors and
calls the library; it computes nothing of the method itself.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

from . import _lib, synth


@dataclasses.dataclass
class Proj:
    fmt: int
    q: torch.Tensor
    scales: torch.Tensor
    scale_2: Optional[torch.Tensor] = None
    mx_scales: Optional[torch.Tensor] = None  # the e8m0 codes an NVFP4 projection came from

    def c(self) -> _lib.qk_weight:
        return _lib.make_weight(self.fmt, self.q, self.scales, self.scale_2)

    def nbytes(self, experts: int = 1) -> int:
        per = (self.q[0].numel() + self.scales[0].numel())
        return per * experts


@dataclasses.dataclass
class DeviceLayer:
    gate: Proj
    up: Proj
    down: Proj

    def c(self) -> _lib.qk_moe_layer:
        return _lib.make_layer(self.gate.c(), self.up.c(), self.down.c())

    @property
    def E(self):
        return self.gate.q.shape[0]

    def expert_bytes(self) -> int:
        """Packed bytes of one expert (three projections, nibbles + scales)."""
        return sum(p.q[0].numel() + p.scales[0].numel() for p in (self.gate, self.up, self.down))


def mx_proj(seed: int, layer: int, proj: int, E: int, rows: int, cols: int, lo: int, hi: int,
            device="cuda") -> Proj:
    q, s = synth.mx_expert_bytes(seed, layer, proj, rows, cols, lo, hi, None, E, device)
    return Proj(_lib.QK_FMT_MXFP4, q, s)


def to_nvfp4(p: Proj, stream=None) -> Proj:
    """Scale-only conversion by the library (nibble tensor shared, not copied)."""
    E, N, K32 = p.scales.shape
    e4 = torch.empty((E, N, 2 * K32), dtype=torch.uint8, device=p.scales.device)
    s2 = torch.empty(E, dtype=torch.float32, device=p.scales.device)
    bad = torch.zeros(1, dtype=torch.int64, device=p.scales.device)
    _lib.quant_convert_mxfp4_to_nvfp4(p.scales, e4, s2, bad, stream)
    return Proj(_lib.QK_FMT_NVFP4, p.q, e4, s2, mx_scales=p.scales)


def nv_proj(seed: int, layer: int, proj: int, E: int, rows: int, cols: int, codes,
            device="cuda") -> Proj:
    """A general NVFP4 projection; ``codes`` = (lo, hi) of its e4m3 block-scale codes."""
    q, s, s2 = synth.nv_expert_bytes(seed, layer, proj, rows, cols, None, E, device, *codes)
    return Proj(_lib.QK_FMT_NVFP4, q, s, s2)


def make_layer(wl: synth.Workload, seed: int = 0, layer: int = 0, fmts=None,
               device="cuda", nv_codes=None) -> DeviceLayer:
    """One MoE layer of workload ``wl``; ``fmts`` = (gate, up, down) formats.

    NVFP4 projections are the MXFP4 ones converted when ``nv_codes`` is None,
    else general NVFP4 sources with e4m3 block-scale codes in ``nv_codes``.
    """
    shapes = ((wl.I, wl.H), (wl.I, wl.H), (wl.H, wl.I))
    if fmts is None:
        f = _lib.QK_FMT_NVFP4 if wl.fmt == "nv" else _lib.QK_FMT_MXFP4
        fmts = (f, f, f)
    projs: List[Proj] = []
    for pi, ((rows, cols), fmt) in enumerate(zip(shapes, fmts)):
        if fmt == _lib.QK_FMT_NVFP4 and nv_codes is not None:
            projs.append(nv_proj(seed, layer, pi, wl.E, rows, cols, nv_codes, device))
            continue
        p = mx_proj(seed, layer, pi, wl.E, rows, cols, wl.code_lo, wl.code_hi, device)
        projs.append(to_nvfp4(p) if fmt == _lib.QK_FMT_NVFP4 else p)
    return DeviceLayer(*projs)


@dataclasses.dataclass
class Fp8Shared:
    wg: torch.Tensor
    sg: torch.Tensor
    wu: torch.Tensor
    su: torch.Tensor
    wd: torch.Tensor
    sd: torch.Tensor

    def nbytes(self) -> int:
        return sum(t.numel() for t in (self.wg, self.sg, self.wu, self.su, self.wd, self.sd))


def make_fp8_shared(seed: int, layer: int, H: int, I: int, device="cuda", block: int = 128) -> Fp8Shared:
    """Shared expert gate/up [I][H], down [H][I]: e4m3 codes uniform over the
    254 non-NaN codes, UE8M0 exponents uniform in 2^-9..2^0, one per
    block x block tile (128, or 32 for the V4.1 layout)."""
    out = []
    for pi, (rows, cols) in zip((synth.TID.SH_GATE, synth.TID.SH_UP, synth.TID.SH_DOWN),
                                ((I, H), (I, H), (H, I))):
        w = synth.fp8_codes(seed, synth.TID.of(layer, pi, 0), rows * cols, device).view(rows, cols)
        s = synth.scale_codes(seed, synth.TID.of(layer, pi, 1), (rows // block) * (cols // block),
                              118, 127, device).view(rows // block, cols // block)
        out += [w, s]
    return Fp8Shared(*out)
