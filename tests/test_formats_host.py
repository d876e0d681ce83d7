"""The format conversions' kernel arithmetic against the oracle, on the CPU (no GPU needed).

``tests/formats_host_emu.cpp`` compiles the per-element functions the CUDA kernels are built from
(``csrc/formats.cuh``) for the host, with IEEE arithmetic and no fused multiply-adds.  Every result must equal
the oracle's bit for bit:
- the E4M3 and E2M1 rounding of dense grids, midpoints included;
- double quantization of random, ragged, constant and power-of-two inputs;
- NVFP4 quantization of random weights, of the format's own grid and of zero blocks.

This pins the kernels' arithmetic before any GPU run.  The GPU parity tests then check the kernels' indexing
and launches on the device.
"""

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import double_quant as D
from oracle import nvfp4 as F

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("emu") / "libfmt_emu.so")
    subprocess.run([cxx, "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-o", out,
                    os.path.join(HERE, "formats_host_emu.cpp")], check=True)
    L = ctypes.CDLL(out)
    f32p, u8p = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_uint8)
    L.emu_e4m3_code.restype, L.emu_e4m3_code.argtypes = ctypes.c_uint32, [ctypes.c_float]
    L.emu_e4m3_value.restype, L.emu_e4m3_value.argtypes = ctypes.c_float, [ctypes.c_uint32]
    L.emu_e2m1_code.restype, L.emu_e2m1_code.argtypes = ctypes.c_uint32, [ctypes.c_float]
    L.emu_e2m1_value.restype, L.emu_e2m1_value.argtypes = ctypes.c_float, [ctypes.c_uint32]
    L.emu_dq_level.restype, L.emu_dq_level.argtypes = ctypes.c_float, [ctypes.c_uint32]
    L.emu_dq_quantize.restype = None
    L.emu_dq_quantize.argtypes = [f32p, ctypes.c_longlong, u8p, f32p, f32p]
    L.emu_dq_dequantize.restype = None
    L.emu_dq_dequantize.argtypes = [u8p, f32p, ctypes.c_float, ctypes.c_longlong, f32p]
    L.emu_nvfp4_quantize.restype = None
    L.emu_nvfp4_quantize.argtypes = [f32p, ctypes.c_longlong, u8p, u8p, f32p]
    L.emu_nvfp4_dequantize.restype = None
    L.emu_nvfp4_dequantize.argtypes = [u8p, u8p, ctypes.c_float, ctypes.c_longlong, f32p]
    return L


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def dq_emu(L, c):
    c = np.ascontiguousarray(c, dtype=np.float32)
    nb = c.size
    code8 = np.zeros(nb, np.uint8)
    c1 = np.zeros((nb + 255) // 256, np.float32)
    mu = np.zeros(1, np.float32)
    L.emu_dq_quantize(_p(c, ctypes.c_float), nb, _p(code8, ctypes.c_uint8), _p(c1, ctypes.c_float),
                      _p(mu, ctypes.c_float))
    back = np.zeros(nb, np.float32)
    L.emu_dq_dequantize(_p(code8, ctypes.c_uint8), _p(c1, ctypes.c_float), float(mu[0]), nb, _p(back, ctypes.c_float))
    return code8, c1, mu[0], back


def fp4_emu(L, w):
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    codes = np.zeros(w.size // 2, np.uint8)
    scales = np.zeros(w.size // 16, np.uint8)
    S = np.zeros(1, np.float32)
    L.emu_nvfp4_quantize(_p(w, ctypes.c_float), w.size, _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8),
                         _p(S, ctypes.c_float))
    back = np.zeros(w.size, np.float32)
    L.emu_nvfp4_dequantize(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), float(S[0]), w.size,
                           _p(back, ctypes.c_float))
    return codes, scales, S[0], back


# ------------------------------------------------------------------ element formats


def test_e4m3_values_and_levels(emu):
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert np.float32(emu.emu_e4m3_value(c)) == np.float32(D.e4m3_value(c)), c
        assert np.float32(emu.emu_dq_level(c)).view(np.uint32) == D.dq_levels()[c].view(np.uint32), c


def test_e4m3_rounding_dense(emu):
    mags = np.array([D.e4m3_value(c) for c in range(0x7F)])
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    t = np.concatenate([np.random.default_rng(0).uniform(0, 470, 20000), np.random.default_rng(1).uniform(0, 0.02, 5000),
                        mids, np.nextafter(mids, np.float32(1e9)), np.nextafter(mids, np.float32(0)), mags,
                        [0.0, 448.0, 463.99, 464.0, 464.01, 1e6, 2.0 ** -6, 2.0 ** -6 - 2.0 ** -11]]).astype(np.float32)
    t = np.maximum(t, 0).astype(np.float32)
    ours = np.array([emu.emu_e4m3_code(float(x)) for x in t], dtype=np.uint8)
    assert np.array_equal(ours, F.e4m3_code_of_nonneg(t))


def test_e2m1_values_and_rounding_dense(emu):
    for c in range(16):
        v = np.float32(emu.emu_e2m1_value(c))
        assert v.view(np.uint32) == np.float32(F.e2m1_value(c)).view(np.uint32), c
    mags = F.e2m1_table()[:8]
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    n = np.concatenate([np.random.default_rng(2).uniform(-8, 8, 20000), mids, -mids, np.nextafter(mids, np.float32(9)),
                        np.nextafter(mids, np.float32(-9)), mags, -mags, [0.0, -0.0, 6.0, 6.5, -100.0]]).astype(np.float32)
    ours = np.array([emu.emu_e2m1_code(float(x)) for x in n], dtype=np.uint8)
    assert np.array_equal(ours, F.e2m1_code_of(n))


# ------------------------------------------------------------------ double quantization


@pytest.mark.parametrize("nb,seed", [(1, 0), (255, 1), (256, 2), (257, 3), (256 * 7 + 19, 4), (65536, 5)])
def test_double_quantization_bit_exact(emu, nb, seed):
    c = np.random.default_rng(seed).uniform(0.005, 0.09, nb).astype(np.float32)
    code8, c1, mu, back = dq_emu(emu, c)
    q, c1o, muo = D.dq_quantize(c)
    assert mu.view(np.uint32) == np.float32(muo).view(np.uint32)
    assert np.array_equal(code8, q)
    assert np.array_equal(c1.view(np.uint32), c1o.view(np.uint32))
    assert np.array_equal(back.view(np.uint32), D.dq_dequantize(q, c1o, muo).view(np.uint32))


def test_double_quantization_of_real_absmax(emu):
    """The constants of an NF4-quantized N(0, 0.015^2) weight (their actual distribution)."""
    from oracle import nf4 as O
    W = (np.random.default_rng(6).standard_normal((96, 4096)) * 0.015).astype(np.float32)
    _, absmax = O.nf4_quantize(W)
    code8, c1, mu, back = dq_emu(emu, absmax)
    q, c1o, muo = D.dq_quantize(absmax)
    assert np.array_equal(code8, q) and np.array_equal(c1, c1o) and mu == muo
    assert np.array_equal(back, D.dq_dequantize(q, c1o, muo))


def test_double_quantization_special_inputs(emu):
    k = np.arange(15)
    for c in (np.full(700, 0.0371, np.float32),                                           # constant: c1 = 0
              np.concatenate([1 + 2.0 ** -k / 2, 1 - 2.0 ** -k / 2]).astype(np.float32),   # exact levels
              np.zeros(300, np.float32)):                                                # all-zero constants
        code8, c1, mu, back = dq_emu(emu, c)
        q, c1o, muo = D.dq_quantize(c)
        assert np.array_equal(code8, q) and np.array_equal(c1, c1o) and mu == muo
        assert np.array_equal(back.view(np.uint32), D.dq_dequantize(q, c1o, muo).view(np.uint32))


# ------------------------------------------------------------------ NVFP4


@pytest.mark.parametrize("rows,cols,std,seed", [(1, 16, 0.015, 0), (3, 48, 1.0, 1), (64, 512, 0.015, 2),
                                                (17, 1024, 0.003, 3)])
def test_nvfp4_bit_exact(emu, rows, cols, std, seed):
    W = (np.random.default_rng(seed).standard_normal((rows, cols)) * std).astype(np.float32)
    codes, scales, S, back = fp4_emu(emu, W)
    co, so, So = F.nvfp4_quantize(W)
    assert S.view(np.uint32) == So.view(np.uint32)
    assert np.array_equal(scales, so)
    assert np.array_equal(codes, co)
    assert np.array_equal(back.view(np.uint32), F.nvfp4_dequantize(co, so, So, W.size).view(np.uint32))


def test_nvfp4_grid_zero_blocks_and_signs(emu):
    rng = np.random.default_rng(7)
    W = (rng.standard_normal(40 * 16) * 0.02).astype(np.float32)
    W[32:48] = 0.0                           # a zero block
    W[50] = -0.0                             # a negative zero
    W[60:64] = W[60:64] * 1e-6               # values that round to (signed) zero
    W[5] = 0.5                               # the tensor's largest magnitude
    for w in (W, np.zeros(64, np.float32)):
        codes, scales, S, back = fp4_emu(emu, w)
        co, so, So = F.nvfp4_quantize(w)
        assert S == So and np.array_equal(scales, so) and np.array_equal(codes, co)
        assert np.array_equal(back.view(np.uint32), F.nvfp4_dequantize(co, so, So, w.size).view(np.uint32))
