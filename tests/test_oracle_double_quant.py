"""Pins for the double-quantization oracle (``oracle.double_quant``) against what the format and the mathematics fix.

Each would fail on a plausible mistake:
- a wrong E4M3 decoding (bias, subnormals, the NaN code);
- a rounding that does not take the nearest level, or breaks a tie the wrong way;
- an offset that is not the mean;
- the wrong group size;
- a missing centring, or a scale applied twice.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import double_quant as D
from oracle import nf4 as O


def ulp32(x):
    """Spacing of fp32 values at |x|."""
    x = np.abs(np.asarray(x, dtype=np.float32))
    return np.spacing(x).astype(np.float64)


def constants(nb, seed, lo=0.02, hi=0.08):
    """Positive fp32 block constants, spread like the absmax of N(0, 0.015^2) blocks."""
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, nb).astype(np.float32)


# ------------------------------------------------------------------ the E4M3 level set


def test_e4m3_decoding_matches_torch_float8():
    """Every one of the 256 bit patterns decodes as torch's float8_e4m3fn does (an independent library)."""
    ours = D.e4m3_table()
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[~both_nan], ref[~both_nan])


def test_e4m3_landmarks():
    t = D.e4m3_table()
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.sum(np.isnan(t)) == 2
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0      # largest finite
    assert t[0x01] == 2.0 ** -9                          # smallest subnormal
    assert t[0x08] == 2.0 ** -6                          # smallest normal
    assert t[0x38] == 1.0                                # exponent field 7 = bias
    assert t[0x00] == 0.0 and t[0x80] == 0.0


def test_sorted_levels():
    vals, codes = D.dq_sorted_levels()
    assert vals.size == 253 and np.all(np.diff(vals.astype(np.float64)) > 0)
    assert vals[0] == -1.0 and vals[-1] == 1.0 and vals[126] == 0.0
    assert codes[126] == 0x00 and codes[-1] == 0x7E and codes[0] == 0xFE
    # symmetric: the negative levels mirror the positive ones
    assert np.array_equal(vals[:126][::-1], -vals[127:])


# ------------------------------------------------------------------ nearest-level codes


def test_codes_are_nearest_levels_brute_force():
    """On random n and on every midpoint and its fp32 neighbours: the code is argmin |n - L| (a tie goes low)."""
    vals, codes = D.dq_sorted_levels()
    v = vals.astype(np.float64)
    mids = ((v[:-1] + v[1:]) / 2.0).astype(np.float32)  # fp32 values at or beside each midpoint
    probes = [np.random.default_rng(3).uniform(-1, 1, 20000).astype(np.float32), mids,
              np.nextafter(mids, np.float32(2)), np.nextafter(mids, np.float32(-2)), vals]
    n = np.concatenate(probes)
    got = D.dq_code_of(n)
    dist = np.abs(n.astype(np.float64)[:, None] - v[None, :])
    best = np.argmin(dist, axis=1)  # first (lower) index on a tie
    assert np.array_equal(got, codes[best])


def test_codes_agree_with_torch_e4m3_rounding_away_from_ties():
    """Away from midpoints the nearest level of n is torch's round-to-nearest E4M3 conversion of 448 n."""
    n = np.random.default_rng(5).uniform(-1, 1, 50000).astype(np.float32)
    vals, _ = D.dq_sorted_levels()
    v = vals.astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2.0
    i = np.searchsorted(mids, n.astype(np.float64))
    near = np.minimum(np.abs(n - mids[np.clip(i - 1, 0, mids.size - 1)]), np.abs(n - mids[np.clip(i, 0, mids.size - 1)]))
    far = near > 4 * ulp32(n) + 1e-12
    ref = torch.from_numpy(n.astype(np.float64) * 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref = np.where(ref == 0x80, 0x00, ref)  # -0 and +0 are one level
    got = D.dq_code_of(n)
    assert far.mean() > 0.99
    assert np.array_equal(got[far], ref[far])


# ------------------------------------------------------------------ the offset


def test_offset_is_the_mean_to_one_rounding():
    """mu is within one fp32 rounding (plus the fp64 sums' error) of the exactly rounded mean."""
    for seed, nb in [(0, 1), (1, 255), (2, 257), (3, 5000)]:
        c = constants(nb, seed)
        mu = D.dq_offset(c)
        exact = math.fsum(float(x) for x in c) / nb
        assert abs(float(mu) - exact) <= 0.5 * ulp32(np.float32(exact)) * (1 + 1e-6) + 1e-15


def test_offset_exact_on_dyadic_constants():
    """Constants that are small multiples of 2^-10: every fp64 sum is exact, so mu = fl32(exact mean)."""
    rng = np.random.default_rng(4)
    c = (rng.integers(1, 200, 1000) / 1024.0).astype(np.float32)
    mean = sum(Fraction(float(x)) for x in c) / len(c)
    assert D.dq_offset(c) == np.float32(float(mean))


# ------------------------------------------------------------------ quantize / dequantize


def test_group_size_from_one_outlier_per_group():
    """One large constant per 256 among nearly equal ones: with groups of 256 each group's scale is set by its
    outlier, so only the outlier reaches |n| >= 1/2 (and it sits on the level +-1).  Groups of 64 would give
    every 64-block its own scale and four such codes per 256."""
    ng = 13
    rng = np.random.default_rng(7)
    c = (0.04 + rng.uniform(-1e-3, 1e-3, 256 * ng)).astype(np.float32)
    pos = rng.integers(0, 256, ng) + 256 * np.arange(ng)
    c[pos] = np.float32(0.08)
    code8, c1, mu = D.dq_quantize(c)
    assert c1.size == ng
    big = np.abs(D.dq_levels()[code8]) >= 0.5
    for g in range(ng):
        assert np.flatnonzero(big[g * 256:(g + 1) * 256]).tolist() == [pos[g] - 256 * g]
    assert np.all(code8[pos] == 0x7E)


def test_error_bound():
    """|absmax' - absmax| <= half the level gap at n times c1, plus the roundings of d, n, the product and the sum."""
    c = constants(256 * 20 + 17, 8)
    code8, c1, mu = D.dq_quantize(c)
    back = D.dq_dequantize(code8, c1, mu).astype(np.float64)
    vals, _ = D.dq_sorted_levels()
    v = vals.astype(np.float64)
    gap = np.max(np.diff(v))  # the widest gap (at |n| near 1): 32 / 448
    scale = np.repeat(c1, 256)[:c.size].astype(np.float64)
    bound = 0.5 * gap * scale + 6 * ulp32(c) + 2 * ulp32(scale)
    assert np.all(np.abs(back - c) <= bound)
    # and the bound is not vacuous: the error is of the order of the level gaps, far below c itself
    assert np.max(np.abs(back - c) / c) < 0.05


def test_constant_input_is_exact():
    """All constants equal: mu is that value, every d is 0, c1 = 0, codes 0x00, and dequantization returns it."""
    c = np.full(700, 0.0371, dtype=np.float32)
    code8, c1, mu = D.dq_quantize(c)
    assert mu == c[0] and not np.any(c1) and not np.any(code8)
    assert np.array_equal(D.dq_dequantize(code8, c1, mu).view(np.uint32), c.view(np.uint32))


def test_power_of_two_scaling_is_exact():
    """Scaling every constant by 2^k scales mu and c1 by 2^k and leaves the codes unchanged."""
    c = constants(256 * 3 + 5, 9)
    q0, c10, mu0 = D.dq_quantize(c)
    q1, c11, mu1 = D.dq_quantize((c * np.float32(8.0)).astype(np.float32))
    assert np.array_equal(q0, q1)
    assert np.array_equal(c11, c10 * np.float32(8.0)) and mu1 == mu0 * np.float32(8.0)


def test_roundtrip_of_power_of_two_levels():
    """The levels that are powers of two are the E4M3 values 7 * 2^j (mantissa field 6): L = +-2^-k, k = 0..14.
    Constants 1 +- 2^-k / 2 (exact in fp32, mean exactly 1, largest |d| = 1/2) must take exactly those codes --
    sign bit, exponent field 15 - k, mantissa field 6 -- and dequantize back bit for bit."""
    k = np.arange(15)
    c = np.concatenate([1 + 2.0 ** -k / 2, 1 - 2.0 ** -k / 2]).astype(np.float32)
    code8, c1, mu = D.dq_quantize(c)
    assert mu == 1.0 and c1[0] == 0.5
    want = np.concatenate([((15 - k) << 3) | 6, 0x80 | ((15 - k) << 3) | 6]).astype(np.uint8)
    assert np.array_equal(code8, want)
    assert np.array_equal(D.dq_dequantize(code8, c1, mu).view(np.uint32), c.view(np.uint32))


def test_dequantize_rejects_nan_codes():
    with pytest.raises(ValueError):
        D.dq_dequantize(np.array([0x7F], np.uint8), np.array([1.0], np.float32), 0.0)


def test_dq_weight_is_nf4_with_rescaled_blocks():
    """The double-quantized weight is the NF4 weight with each block scaled by absmax' / absmax (codes unchanged)."""
    rng = np.random.default_rng(11)
    N, K = 8, 512
    W = (rng.standard_normal((N, K)) * 0.015).astype(np.float32)
    codes, absmax = O.nf4_quantize(W)
    code8, c1, mu = D.dq_quantize(absmax)
    w_dq = D.nf4_dequantize_dq(codes, code8, c1, mu, N * K).reshape(-1, 64).astype(np.float64)
    w = O.nf4_dequantize(codes, absmax, N * K).reshape(-1, 64).astype(np.float64)
    ratio = (D.dq_dequantize(code8, c1, mu).astype(np.float64) / absmax.astype(np.float64))[:, None]
    assert np.allclose(w_dq, w * ratio, rtol=2 ** -22, atol=0)


@pytest.mark.parametrize("mistake", ["no_centring", "scale_twice", "wrong_sign"])
def test_planted_mistakes_fail_the_error_bound(mistake):
    c = constants(256 * 4, 12)
    code8, c1, mu = D.dq_quantize(c)
    if mistake == "no_centring":
        back = D.dq_dequantize(code8, c1, 0.0)
    elif mistake == "scale_twice":
        back = D.dq_dequantize(code8, c1 * c1, mu)
    else:
        back = D.dq_dequantize(code8 ^ np.uint8(0x80), c1, mu)
    vals, _ = D.dq_sorted_levels()
    gap = np.max(np.diff(vals.astype(np.float64)))
    scale = np.repeat(c1, 256)[:c.size].astype(np.float64)
    bound = 0.5 * gap * scale + 6 * ulp32(c) + 2 * ulp32(scale)
    assert not np.all(np.abs(back.astype(np.float64) - c) <= bound)
