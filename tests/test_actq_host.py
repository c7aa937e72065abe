"""The activation-quantization arithmetic of the block-scaled paths
(block_quantized_expert_mxfp4_b200/csrc/qk_actq.cuh), compiled for the host by
nvcc, against the oracle's quantizer: scale codes and element values bit for
bit, on bf16 (x) and fp32 (h) blocks with exact ties, near-ties, zero,
subnormal and extreme blocks.  No GPU: the same source the kernels include."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from conftest import ROOT
from ref_decode import E2M1, E4M3

CSRC = os.path.join(ROOT, "block_quantized_expert_mxfp4_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "native", "actq_host.cu")
OUT = os.path.join(ROOT, "tests", "_build", "libactq_host.so")


@pytest.fixture(scope="module")
def host():
    nvcc = os.environ.get("NVCC", shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc")
    deps = [SRC, os.path.join(CSRC, "qk_actq.cuh")]
    if not os.path.exists(OUT) or os.path.getmtime(OUT) < max(map(os.path.getmtime, deps)):
        os.makedirs(os.path.dirname(OUT), exist_ok=True)
        subprocess.check_call([nvcc, "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I", CSRC,
                               "-I", os.path.join(ROOT, "include"), SRC, "-o", OUT])
    L = ctypes.CDLL(OUT)
    L.actq_host.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    L.actq_host_fp4packed.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    L.actq_host_nv_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]
    L.actq_host_nv_code.argtypes = [ctypes.c_int]
    L.actq_host_nv_code.restype = ctypes.c_uint
    L.actq_host_pow2.argtypes = [ctypes.c_int]
    L.actq_host_pow2.restype = ctypes.c_float

    def run(v, fp4):
        v = np.ascontiguousarray(v, np.float32)
        codes = np.empty(v.size, np.uint8)
        scales = np.empty(v.size // 32, np.uint8)
        L.actq_host(v.ctypes.data, v.size, int(fp4), codes.ctypes.data, scales.ctypes.data)
        return codes, scales

    def packed(v):
        v = np.ascontiguousarray(v, np.float32)
        p = np.empty(v.size // 2, np.uint8)
        scales = np.empty(v.size // 32, np.uint8)
        L.actq_host_fp4packed(v.ctypes.data, v.size, p.ctypes.data, scales.ctypes.data)
        return p, scales
    def nv_rows(v):
        v = np.ascontiguousarray(v, np.float32)
        rows, n = v.shape
        p = np.empty((rows, n // 2), np.uint8)
        codes = np.empty((rows, n // 32), np.uint8)
        fac = np.empty(rows, np.float32)
        L.actq_host_nv_rows(v.ctypes.data, rows, n, p.ctypes.data, codes.ctypes.data, fac.ctypes.data)
        return p, codes, fac
    run.packed = packed
    run.nv_rows = nv_rows
    run.lib = L
    return run


def _bf16(a):
    u = np.asarray(a, np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).view(np.float32)


def _blocks():
    rng = np.random.default_rng(0)
    out = []
    for trial in range(400):
        v = rng.standard_normal(32) * 2.0 ** rng.integers(-4, 5, 32) * 2.0 ** rng.integers(-60, 60)
        out.append(v)
    # exact ties and near-ties of both grids: multiples of quarter steps, and
    # the same values one fp32 ulp away
    for top in (6.0, 448.0):
        base = np.linspace(-top, top, 32 * 8).reshape(-1, 32)
        for b in base:
            b = b.copy()
            b[0] = top * 1.25  # block maximum in the top binade of the rule
            out += [b, np.nextafter(b.astype(np.float32), np.float32(np.inf)),
                    np.nextafter(b.astype(np.float32), np.float32(-np.inf))]
    # every midpoint of each grid, in blocks whose maximum (4, or 256) puts
    # the scale at 2^0 for that format, both signs, and scaled by 2^-20
    for grid, anchor in ((E2M1[:8], 4.0), (np.unique(E4M3[:0x7F]), 256.0)):
        mids = (grid[:-1] + grid[1:]) / 2
        mids = mids[mids < anchor]
        for i in range(0, mids.size, 15):
            chunk = mids[i:i + 15]
            blk = np.zeros(32)
            blk[0] = anchor
            blk[1:1 + chunk.size] = chunk
            blk[16:16 + chunk.size] = -chunk
            out += [blk, blk * 2.0 ** -20]
    out.append(np.zeros(32))
    out.append(np.full(32, 2.0 ** -140))                  # fp32 subnormals
    out.append(np.r_[3.0e38, -1.0, np.zeros(30)])        # near fp32 max
    out.append(np.r_[2.0 ** -126, 2.0 ** -149, np.zeros(30)])
    return np.concatenate(out).astype(np.float32)


@pytest.mark.parametrize("fp4", [0, 1])
@pytest.mark.parametrize("kind", ["fp32", "bf16"])
def test_matches_oracle_bit_for_bit(host, fp4, kind):
    v = _blocks()
    if kind == "bf16":
        v = _bf16(v)
    codes, scales = host(v, fp4)
    oc, os_, _ = oracle.act_quant(v.astype(np.float64), oracle.ACT_MXFP4 if fp4 else oracle.ACT_E4M3)
    assert np.array_equal(scales, os_)
    if fp4:  # the device writes the e2m1 value as an e4m3 code
        got, want = E4M3[codes], E2M1[oc]
        assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))
    else:
        assert np.array_equal(codes, oc)


@pytest.mark.parametrize("kind", ["fp32", "bf16"])
def test_packed_e2m1_matches_oracle_codes(host, kind):
    """The packed form the fp4 x fp4 tensor core reads (QK_ACT_MXFP4 tiles):
    every nibble is the oracle's e2m1 code (sign included) and every scale its
    e8m0 code; element 2 i sits in the low nibble of byte i, as in the packed
    weights."""
    v = _blocks()
    if kind == "bf16":
        v = _bf16(v)
    p, scales = host.packed(v)
    oc, os_, _ = oracle.act_quant(v.astype(np.float64), oracle.ACT_MXFP4)
    nib = np.empty(v.size, np.uint8)
    nib[0::2], nib[1::2] = p & 0xF, p >> 4
    assert np.array_equal(scales, os_)
    assert np.array_equal(nib, oc)



def test_nv_scale_code_is_the_e4m3_power_of_two(host):
    """The ue4m3 code of 2^d that the NVFP4 fp4-mode tiles carry, for every d
    the rule produces, against the ml_dtypes e4m3 decoder: exact for
    -9 <= d <= 8 (subnormals 2^-9 .. 2^-7 included), 0 below."""
    for d in range(-20, 9):
        code = host.lib.actq_host_nv_code(d)
        if d >= -9:
            assert E4M3[code] == 2.0 ** d, (d, code)
        else:
            assert code == 0, (d, code)
    for e in range(-149, 128):
        assert float(host.lib.actq_host_pow2(e)) == 2.0 ** e, e


def test_nv_rows_restore_the_mxfp4_scales(host):
    """Per row: the packed codes are the MXFP4 mode's (the oracle's), and
    every 32-block within 17 binades of the row's largest scale gets an
    e4m3 code whose value times the row factor is 2^(c - 127) exactly (c the
    oracle's e8m0 code); blocks further below get code 0 (dropped)."""
    rng = np.random.default_rng(7)
    rows = []
    for r in range(24):
        v = rng.standard_normal(512) * 2.0 ** rng.integers(-30, 30)
        # blocks scaled down by up to 2^-40 (some far below the row's largest)
        v *= np.repeat(2.0 ** -rng.integers(0, 41, 16), 32)
        if r % 5 == 0:
            v[32:64] = 0.0  # an all-zero block
        rows.append(v)
    v = np.asarray(rows, np.float32)
    p, codes, fac = host.nv_rows(v)
    for r in range(v.shape[0]):
        oc, osc, _ = oracle.act_quant(v[r].astype(np.float64), oracle.ACT_MXFP4)
        pm, sm = host.packed(v[r])
        assert np.array_equal(p[r], pm)
        assert np.array_equal(np.asarray(osc, np.uint8), sm)
        cmax = int(np.max(sm))
        assert float(fac[r]) == 2.0 ** (cmax - 135)
        for b, c in enumerate(sm.astype(int)):
            if c >= cmax - 17:
                assert E4M3[codes[r, b]] * float(fac[r]) == 2.0 ** (c - 127), (r, b, c, cmax)
            else:
                assert codes[r, b] == 0, (r, b, c, cmax)
