"""The NVFP4 -> MXFP4 block rule of the library
(block_quantized_expert_mxfp4_b200/csrc/qk_convert_nv.h), compiled for the
host by nvcc, against the oracle's conversion: every pair of non-NaN e4m3
codes under several scale_2 values (powers of two, not, fp32 subnormal, huge,
negative), codes and inexact counts bit for bit.  No GPU: the kernel calls the
same function."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from conftest import ROOT

CSRC = os.path.join(ROOT, "block_quantized_expert_mxfp4_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "native", "convert_nv_host.cu")
OUT = os.path.join(ROOT, "tests", "_build", "libconvert_nv_host.so")
CODES = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)


@pytest.fixture(scope="module")
def host():
    nvcc = os.environ.get("NVCC", shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc")
    deps = [SRC, os.path.join(CSRC, "qk_convert_nv.h")]
    if not os.path.exists(OUT) or os.path.getmtime(OUT) < max(map(os.path.getmtime, deps)):
        os.makedirs(os.path.dirname(OUT), exist_ok=True)
        subprocess.check_call([nvcc, "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I", CSRC,
                               "-I", os.path.join(ROOT, "include"), SRC, "-o", OUT])
    L = ctypes.CDLL(OUT)
    L.convert_nv_host.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int] + [ctypes.c_void_p] * 3

    def run(pairs, s2):
        pairs = np.ascontiguousarray(pairs, np.uint8)
        s2 = np.ascontiguousarray(s2, np.float32)
        n = s2.size
        out = np.empty(n, np.uint8)
        bad, nn = ctypes.c_ulonglong(0), ctypes.c_int(0)
        L.convert_nv_host(pairs.ctypes.data, s2.ctypes.data, n, out.ctypes.data, ctypes.byref(bad),
                          ctypes.byref(nn))
        return out, bad.value, nn.value
    return run


@pytest.mark.parametrize("s2", [1.0, 2.0 ** -9, 0.75, 0.1, 2.0 ** -130, 3.0e38, -1.0, 2.0 ** 100])
def test_every_code_pair_matches_oracle(host, s2):
    a, b = np.meshgrid(CODES, CODES, indexing="ij")
    pairs = np.stack([a.reshape(-1), b.reshape(-1)], 1)          # [n][2]
    scales = np.full(pairs.shape[0], s2, np.float32)
    got, bad, nn = host(pairs, scales)
    want, wbad = oracle.convert_nv_to_mx(pairs.reshape(1, -1, 2), np.array([s2], np.float32))
    assert nn == 0
    assert np.array_equal(got, want.reshape(-1)) and bad == wbad


def test_nan_codes_write_255(host):
    pairs = np.array([[0x38, 0x7F], [0xFF, 0x38], [0x38, 0x38]], np.uint8)
    got, bad, nn = host(pairs, np.ones(3, np.float32))
    assert list(got) == [255, 255, 127] and nn == 2 and bad == 0
