"""How much of the GEMM tolerance the fused kernels' in-register dequantization uses (CPU only).

Inside the fused GEMMs a weight is expanded as the bf16 product of the bf16-rounded level and the bf16-rounded
block scale, not as the exact fp32 product rounded once.  This test emulates that rounding independently (numpy
bit manipulation, no library code) at the bench layer's contraction length and checks that its effect on the
forward and dX products stays far inside the tolerance the GPU results are held to -- so a parity failure on the
GPU cannot be blamed on this design choice alone.
"""

import numpy as np

from oracle import linear as L
from oracle import nf4 as O


def bf16_round(a):
    """Round fp32 values to bf16 (round to nearest, ties to even) and return them as fp64."""
    b = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def kernel_weight(codes, absmax, N, K):
    """bf16(bf16(level) * bf16(absmax)): the product of two bf16 values is exact in fp32, then rounded to bf16."""
    lev = O.nf4_codebook()[O.nf4_unpack(codes)].reshape(N, K)
    sc = np.repeat(absmax, 64).reshape(N, K)
    prod = (bf16_round(lev) * bf16_round(sc)).astype(np.float32)  # exact: 8-bit x 8-bit significands
    return bf16_round(prod)


def test_in_register_dequantization_uses_a_small_part_of_the_tolerance():
    rng = np.random.default_rng(0)
    M, N, K = 64, 256, 4096
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, absmax = O.nf4_quantize(W)
    exact = L.dequantized_weight(codes, absmax, N, K)
    approx = kernel_weight(codes, absmax, N, K)
    # per element: within three bf16 roundings of the exact value
    rel = np.abs(approx - exact) / np.maximum(np.abs(exact), 1e-30)
    assert np.max(rel[exact != 0]) <= 3 * 2.0 ** -8
    x = bf16_round(rng.standard_normal((M, K)))
    dy = bf16_round(rng.standard_normal((M, N)))
    fwd = L.compare(x @ approx.T, x @ exact.T)
    dxr = L.compare(dy @ approx, dy @ exact)
    # The GPU is held to rel_fro <= 1e-2 and max-abs <= 2e-2 max|ref|.  For products of random-sign terms the
    # relative error is about the per-element rms error (~1.2 * 2^-9 = 2.5e-3): under 40% of the tolerance.
    for res in (fwd, dxr):
        assert res["rel_fro"] < 4e-3 and res["max_abs_frac"] < 1e-2, res
