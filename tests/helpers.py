"""Shared test helpers: oracle sub-layers regenerated on the host from the
seeded generators, and the parity metrics."""
import json
import os

import numpy as np
import torch

import oracle
from block_quantized_expert_mxfp4_b200 import synth

MX, NV = 1, 2
TOL_REL = 5e-3      # max|gpu - oracle| / max|oracle|
TOL_COS = 0.9999


def oracle_sublayer(wl, seed, layer, experts, fmts=(MX, MX, MX), nv_codes=None):
    """oracle.Layer holding only `experts` (in that order), bytes regenerated
    on the host; NVFP4 projections converted by the oracle's own rule, or, with
    `nv_codes`, the general NVFP4 source drawn with those block-scale codes."""
    shapes = ((wl.I, wl.H), (wl.I, wl.H), (wl.H, wl.I))
    ws = []
    for pi, ((rows, cols), fmt) in enumerate(zip(shapes, fmts)):
        if fmt == NV and nv_codes is not None:
            q, e4, s2 = synth.nv_expert_bytes(seed, layer, pi, rows, cols, list(experts), wl.E,
                                              "cpu", *nv_codes)
            ws.append(oracle.Weight(NV, q, e4, s2))
            continue
        q, s = synth.mx_expert_bytes(seed, layer, pi, rows, cols, wl.code_lo, wl.code_hi,
                                     list(experts), wl.E, "cpu")
        if fmt == NV:
            e4, s2, bad = oracle.convert_mx_to_nv(s)
            assert bad == 0
            ws.append(oracle.Weight(NV, q, e4, s2))
        else:
            ws.append(oracle.Weight(MX, q, s))
    return oracle.Layer(*ws)


def oracle_moe(wl, seed, layer, x_bf16, ids, w, fmts=(MX, MX, MX), nv_codes=None):
    """Oracle y for tokens x with routing (ids, w): experts remapped to a sub-layer."""
    ids = np.asarray(ids)
    experts = sorted(set(int(e) for e in ids.reshape(-1)))
    remap = {e: i for i, e in enumerate(experts)}
    L = oracle_sublayer(wl, seed, layer, experts, fmts, nv_codes)
    sub = np.vectorize(remap.get)(ids).astype(np.int32)
    return oracle.moe_forward(L, x_bf16, sub, np.asarray(w, dtype=np.float64))


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def cosine(got, ref):
    a = np.asarray(got, dtype=np.float64).reshape(-1)
    b = np.asarray(ref, dtype=np.float64).reshape(-1)
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def assert_parity(got, ref, tol=TOL_REL, cos=TOL_COS, what=""):
    e, c = rel_err(got, ref), cosine(got, ref)
    log = os.environ.get("QK_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"case": what, "max_rel": e, "cosine": c, "tol": tol}) + "\n")
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), what
    assert e <= tol and c >= cos, f"{what}: max-rel {e:.3e} (tol {tol}), cosine {c:.7f}"
    return e, c


# ------------------------------------------- activation-quantized modes --

def _grid(aq):
    """Positive values of the activation element grid of mode aq."""
    import ml_dtypes
    if aq == oracle.ACT_MXFP4:
        v = np.arange(8, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    else:
        v = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return np.unique(v)


def _quant_at(v, X, aq):
    """Elements of one block quantized with the scale 2^X given (RNE to the
    grid, saturating): the alternative of a block whose scale is ambiguous."""
    g = _grid(aq)
    q = np.abs(v) / 2.0 ** X
    i = np.clip(np.searchsorted(g, q), 1, g.size - 1)
    lo, hi = g[i - 1], g[i]
    pick_hi = (q - lo > hi - q) | ((q - lo == hi - q) & (i % 2 == 0))  # tie: the even code (index)
    r = np.where(q >= g[-1], g[-1], np.where(pick_hi, hi, lo))
    return np.sign(v) * r * 2.0 ** X


def act_quant_alternatives(h32, hq, aq, eps):
    """Where the code of an fp32 h element is not unique: (index array, the
    other valid dequantized values) pairs.  An element whose scaled value lies
    within a relative eps of a grid midpoint may take the other neighbour; a
    block whose maximum lies within eps of a power of two may take the scale
    one binade away (all its elements together)."""
    g = _grid(aq)
    mids = (g[:-1] + g[1:]) / 2
    emax = 2 if aq == oracle.ACT_MXFP4 else 8
    out = []
    for b in range(h32.size // 32):
        sl = slice(32 * b, 32 * b + 32)
        v = h32[sl]
        amax = np.abs(v).max()
        if amax == 0:
            continue
        _, ex = np.frexp(amax)
        X = max(min(ex - 1 - emax, 127), -127)
        p2 = 2.0 ** (ex - 1)                      # amax in [p2, 2 p2)
        if amax <= p2 * (1 + eps) and X - 1 >= -127:
            out.append((np.arange(sl.start, sl.stop), _quant_at(v, X - 1, aq)))
        if amax >= 2 * p2 * (1 - eps) and X + 1 <= 127:
            out.append((np.arange(sl.start, sl.stop), _quant_at(v, X + 1, aq)))
        q = np.abs(v) / 2.0 ** X
        j = np.clip(np.searchsorted(mids, q), 0, mids.size - 1)
        for jj in (j, np.clip(j - 1, 0, mids.size - 1)):
            near = np.abs(q - mids[jj]) <= eps * np.maximum(q, mids[jj])
            for i in np.nonzero(near)[0]:
                m = mids[jj[i]]
                lo, hi = g[jj[i]], g[jj[i] + 1]
                cur = abs(hq[sl][i]) / 2.0 ** X
                other = hi if cur == lo else lo
                out.append((np.array([sl.start + i]), np.sign(v[i]) * other * 2.0 ** X * np.ones(1)))
    return out


def _down_columns(layer, e, idx):
    """Columns idx of expert e's dequantized down matrix (MXFP4, or NVFP4
    with its scale_2), decoded with the library tables of ml_dtypes:
    [hidden][len(idx)]."""
    from ref_decode import E2M1, E4M3, E8M0
    d = layer.down
    byte = d.q[e][:, idx // 2]
    code = np.where(idx % 2 == 1, byte >> 4, byte & 0x0F)
    if d.fmt == NV:
        return E2M1[code] * E4M3[d.scales[e][:, idx // 16]] * float(d.scale_2[e])
    assert d.fmt == MX
    return E2M1[code] * E8M0[d.scales[e][:, idx // 32]]


def assert_parity_act_quant(y, layer, x_bf16, ids, w, aq, eps=2.0 ** -13, tol=TOL_REL, what=""):
    """Parity of a quantized-activation forward against the oracle run in the
    same mode.  x is bf16, so its codes are unique (both sides decide from the
    same exact values).  h is fp32 on both sides, but its summation order and
    SiLU differ, so an h code is unique only away from its decision
    boundaries: where the oracle's fp32 h lies within a relative eps of a
    grid midpoint (or a block maximum within eps of a power of two), the
    other code is valid too.  The GPU y must equal the oracle's y under some
    choice of such valid codes: the alternatives that best explain the
    difference are taken greedily (least squares, one at a time), then the
    usual bar applies.  Returns (max-rel, cosine, alternatives used, offered)."""
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    yo = oracle.moe_forward(layer, x_bf16, ids, w, aq)
    adj = yo.copy()
    used = offered = 0
    for t in range(ids.shape[0]):
        deltas = []
        for s in range(ids.shape[1]):
            e = int(ids[t, s])
            g, u, hq, _ = oracle.expert_ffn(layer, e, x_bf16[t], aq)
            h32 = (g / (1.0 + np.exp(-g)) * u).astype(np.float32).astype(np.float64)
            for idx, alt in act_quant_alternatives(h32, hq, aq, eps):
                dv = alt - hq[idx]
                if np.any(dv != 0):
                    deltas.append(w[t, s] * (_down_columns(layer, e, idx) @ dv))
        offered += len(deltas)
        r = y[t] - adj[t]
        while deltas:
            gain = [2 * (r @ d) - d @ d for d in deltas]
            i = int(np.argmax(gain))
            if gain[i] <= 0:
                break
            r = r - deltas[i]
            adj[t] += deltas.pop(i)
            used += 1
    e, c = assert_parity(y, adj, tol=tol, what=f"{what} ({used} of {offered} alternative h codes)")
    return e, c, used, offered
