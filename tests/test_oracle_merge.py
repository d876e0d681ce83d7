"""Pins for the LoRA merge oracle (``oracle.merge``) against what the mathematics fixes.

Each test would fail on a plausible mistake: A or B transposed or indexed by the wrong axis, s applied twice
or not at all, a dropped rank term, a merge that perturbs the base when the adapter is zero, a requantization
that does not take the nearest level.
"""

import numpy as np
import pytest
import torch

from oracle import merge as M
from oracle import nf4 as O

U = 2.0 ** -24  # fp32 unit roundoff


def bf16(a):
    return O.round_bf16(np.asarray(a, dtype=np.float32))


def base(N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, absmax = O.nf4_quantize(W)
    return rng, codes, absmax


@pytest.mark.parametrize("which", ["B", "A", "s", "r0"])
def test_zero_adapter_returns_the_base_exactly(which):
    """B = 0, A = 0, s = 0 or r = 0: W' is the dequantized base bit for bit, and requantizing it gives back
    the original codes and scales (quantize after dequantize is the identity: each block's largest element
    sits on the level +-1, so the scale is unchanged, and every other value is a level, far from a midpoint)."""
    N, K, r = 6, 192, 8
    rng, codes, absmax = base(N, K, 1)
    A = bf16(rng.standard_normal((r, K)) * 0.1)
    B = bf16(rng.standard_normal((N, r)) * 0.1)
    s = 2.0
    if which == "B":
        B = np.zeros_like(B)
    elif which == "A":
        A = np.zeros_like(A)
    elif which == "s":
        s = 0.0
    else:
        A, B = np.zeros((0, K), np.float32), np.zeros((N, 0), np.float32)
    d = O.nf4_dequantize(codes, absmax, N * K).reshape(N, K)
    w = M.merge_lora(codes, absmax, A, B, s, N, K)
    assert np.array_equal(w.view(np.uint32), d.view(np.uint32))
    c2, a2 = M.merge_lora_nf4(codes, absmax, A, B, s, N, K)
    assert np.array_equal(c2, codes) and np.array_equal(a2.view(np.uint32), absmax.view(np.uint32))


def test_zero_block_stays_zero():
    N, K = 2, 128
    codes = np.full(N * K // 2, 0x77, np.uint8)  # all-zero blocks (reading R3)
    absmax = np.zeros(N * K // 64, np.float32)
    w = M.merge_lora(codes, absmax, np.zeros((1, K), np.float32), np.zeros((N, 1), np.float32), 3.0, N, K)
    assert not np.any(w)
    c2, a2 = M.merge_lora_nf4(codes, absmax, np.zeros((1, K), np.float32), np.zeros((N, 1), np.float32), 3.0, N, K)
    assert np.array_equal(c2, codes) and not np.any(a2)


def test_hand_expanded_terms():
    """Rank 2 with a few exact non-zero entries: W'[n,k] = d[n,k] + s sum_j B[n,j] A[j,k] written out by hand."""
    N, K = 2, 64
    _, codes, absmax = base(N, K, 2)
    d = O.nf4_dequantize(codes, absmax, N * K).reshape(N, K)
    A = np.zeros((2, K), np.float32)
    A[0, 3], A[1, 10] = 0.25, -1.5
    B = np.array([[1.0, 0.0], [0.5, 2.0]], np.float32)
    s = 2.0
    want = d.copy()
    want[0, 3] = np.float32(d[0, 3]) + np.float32(2.0 * 1.0 * 0.25)      # row 0 takes rank 0 only
    want[1, 3] = np.float32(d[1, 3]) + np.float32(2.0 * 0.5 * 0.25)
    want[1, 10] = np.float32(d[1, 10]) + np.float32(2.0 * 2.0 * -1.5)    # rank 1 reaches row 1 only
    w = M.merge_lora(codes, absmax, A, B, s, N, K)
    assert np.array_equal(w.view(np.uint32), want.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("N,K,r,s", [(5, 128, 1, 2.0), (7, 256, 16, 0.5), (3, 64, 64, 2.0), (4, 128, 200, 1.0)])
def test_error_bound_against_fp64_product(N, K, r, s):
    """Recursive fp32 summation of r exact products, one scaling and one addition: |W' - W'_exact| is at most
    (r + 2) u (|d| + |s| sum_j |B_j A_j|) with u = 2^-24 -- tight enough to catch a wrong or missing term."""
    rng, codes, absmax = base(N, K, N + K + r)
    A = bf16(rng.standard_normal((r, K)) / np.sqrt(K))
    B = bf16(rng.standard_normal((N, r)) * 0.05)
    d = O.nf4_dequantize(codes, absmax, N * K).reshape(N, K).astype(np.float64)
    exact = d + s * (B.astype(np.float64) @ A.astype(np.float64))
    mag = np.abs(d) + abs(s) * (np.abs(B.astype(np.float64)) @ np.abs(A.astype(np.float64)))
    w = M.merge_lora(codes, absmax, A, B, s, N, K).astype(np.float64)
    assert np.all(np.abs(w - exact) <= (r + 2) * U * mag + 1e-30)
    # and the adapter term is really there (not a no-op)
    assert np.max(np.abs(w - d)) > 0.1 * np.max(np.abs(exact - d))


def test_requantized_codes_are_nearest_levels():
    N, K, r, s = 4, 256, 8, 2.0
    rng, codes, absmax = base(N, K, 7)
    A = bf16(rng.standard_normal((r, K)) / np.sqrt(K))
    B = bf16(rng.standard_normal((N, r)) * 0.05)
    w = M.merge_lora(codes, absmax, A, B, s, N, K).reshape(-1, 64)
    c2, a2 = M.merge_lora_nf4(codes, absmax, A, B, s, N, K)
    assert np.array_equal(a2, np.max(np.abs(w), axis=1))
    n = (w.astype(np.float64) / a2[:, None].astype(np.float64)).astype(np.float32).astype(np.float64)
    levels = O.nf4_codebook().astype(np.float64)
    dist = np.abs(n[..., None] - levels[None, None, :])
    best = np.argmin(dist, axis=-1)  # argmin takes the first (lower) index on a tie, as reading R2 does
    assert np.array_equal(O.nf4_unpack(c2).reshape(-1, 64), best.astype(np.uint8))


def test_bf16_output_is_round_to_nearest_even():
    N, K, r = 3, 128, 4
    rng, codes, absmax = base(N, K, 9)
    A = bf16(rng.standard_normal((r, K)))
    B = bf16(rng.standard_normal((N, r)))
    w = M.merge_lora(codes, absmax, A, B, 2.0, N, K)
    bits = M.merge_lora_bf16_bits(codes, absmax, A, B, 2.0, N, K)
    ref = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


@pytest.mark.parametrize("mistake", ["s_twice", "drop_last_rank", "B_transposed_rank"])
def test_planted_mistakes_are_caught(mistake):
    """Wrong merges planted on the CPU must fail the error-bound pin."""
    N, K, r, s = 5, 128, 4, 2.0
    rng, codes, absmax = base(N, K, 11)
    A = bf16(rng.standard_normal((r, K)) / np.sqrt(K))
    B = bf16(rng.standard_normal((N, r)) * 0.05)
    d = O.nf4_dequantize(codes, absmax, N * K).reshape(N, K)
    if mistake == "s_twice":
        bad = d + np.float32(s * s) * (B @ A)
    elif mistake == "drop_last_rank":
        bad = d + np.float32(s) * (B[:, :-1] @ A[:-1])
    else:  # ranks of B taken in reverse order against A
        bad = d + np.float32(s) * (B[:, ::-1] @ A)
    exact = d.astype(np.float64) + s * (B.astype(np.float64) @ A.astype(np.float64))
    mag = np.abs(d) + abs(s) * (np.abs(B.astype(np.float64)) @ np.abs(A.astype(np.float64)))
    assert not np.all(np.abs(bad.astype(np.float64) - exact) <= (r + 2) * U * mag + 1e-30)
