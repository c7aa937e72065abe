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
