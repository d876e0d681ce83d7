"""Pins for the NVFP4 oracle (``oracle.nvfp4``) against what the pages, the formats and the mathematics fix.

Each would fail on a plausible mistake:
- a wrong E2M1 decoding (bias, the subnormal), or a range other than +-6;
- a rounding that is not nearest-even, or does not saturate;
- an E4M3 block scale rounded differently from torch's float8 conversion;
- a missing per-tensor scale;
- the wrong group size;
- the nibble order reversed.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4 as F
from oracle import double_quant as D


def weights(rows, cols, seed, std=0.015):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((rows, cols)) * std).astype(np.float32)


# ------------------------------------------------------------------ E2M1


def test_e2m1_values_and_range():
    """The magnitudes of the 1-sign / 2-exponent / 1-mantissa float, whose largest is 6: the pages give the
    format's range as about +-6 ("Major Unsloth Update: NVFP4 Quantization Export and DeepSeek-V4 Training
    Support", section "NVFP4: A Quantization Format for the Next Generation of Hardware")."""
    t = F.e2m1_table()
    assert t[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(t[8:], -t[:8]) and np.signbit(t[8])
    assert np.max(np.abs(t)) == 6.0


def test_e2m1_rounding_brute_force():
    """Nearest value, a tie to the even mantissa bit, saturation past 6, the sign kept -- on random values, on
    every midpoint and on its fp32 neighbours."""
    t = F.e2m1_table()
    mags = t[:8]
    mids = (mags[:-1] + mags[1:]) / 2
    probe = np.concatenate([np.random.default_rng(1).uniform(-9, 9, 20000), mids, -mids, [6.5, -7.0, 100.0, 0.0],
                            np.nextafter(mids, 10), np.nextafter(mids, -10), mags, -mags]).astype(np.float32)
    got = F.e2m1_code_of(probe)
    for x, c in zip(probe.tolist(), got.tolist()):
        m = min(abs(x), 6.0)
        d = np.abs(mags - m)
        best = np.flatnonzero(d == d.min())
        want = best[0] if best.size == 1 else best[best % 2 == 0][0]  # tie: the even mantissa bit
        assert c & 7 == want, (x, c)
        assert (c >> 3) == (1 if np.signbit(np.float32(x)) else 0), (x, c)


def test_e2m1_ties_by_hand():
    n = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, -0.25], np.float32)
    vals = F.e2m1_table()[F.e2m1_code_of(n)]
    assert vals.tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -4.0, -0.0]


# ------------------------------------------------------------------ E4M3 block scales


def test_e4m3_scale_rounding_matches_torch():
    """Non-negative fp32 values up to 460 (past 448 torch rounds to 448 until 464): nearest-even E4M3."""
    t = np.concatenate([np.random.default_rng(2).uniform(0, 460, 30000),
                        np.random.default_rng(3).uniform(0, 2.0 ** -5, 10000)]).astype(np.float32)
    ours = F.e4m3_code_of_nonneg(t)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_scale_ties_match_torch():
    """Exact midpoints between neighbouring E4M3 values (fp32-exact): ties go to the even mantissa, as torch's."""
    mags = np.array([D.e4m3_value(c) for c in range(0x7F)])
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (mags[:-1] + mags[1:]) / 2)
    ours = F.e4m3_code_of_nonneg(mids)
    ref = torch.from_numpy(mids).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------ quantize / dequantize


def test_worked_tensor_round_trips_exactly():
    """A tensor built on the format's own grid: S = 2^-10 (one block reaches 6 * 448 * 2^-10 = 2.625), block
    scales chosen from normal E4M3 values, each block holding a +-6 element, every element a level times its
    block scale.  Quantization must recover the chosen codes and scales, and dequantization the tensor, bit for
    bit.  The packed bytes also fix the nibble order: element 2j in the low nibble."""
    rng = np.random.default_rng(4)
    nblk = 40
    sb = rng.integers(0x08, 0x7E, nblk).astype(np.uint8)   # normal E4M3 codes below 448
    sb[7] = 0x7E                                           # one block at 448: amax = 2.625
    codes = rng.integers(0, 16, (nblk, 16)).astype(np.uint8)
    codes[:, 3] = 0x7                                      # +6 in every block: its largest magnitude
    codes[codes == 0x8] = 0x0                              # no -0 in the constructed tensor
    S = 2.0 ** -10
    sval = np.array([D.e4m3_value(int(c)) for c in sb])
    w = (F.e2m1_table()[codes] * (sval * S)[:, None]).astype(np.float32).reshape(-1)
    assert np.all(w.astype(np.float64) == (F.e2m1_table()[codes] * (sval * S)[:, None]).reshape(-1))
    got_codes, got_sb, got_S = F.nvfp4_quantize(w)
    assert got_S == np.float32(S)
    assert np.array_equal(got_sb, sb)
    flat = codes.reshape(-1)
    assert np.array_equal(got_codes, (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8))
    assert np.array_equal(F.nvfp4_dequantize(got_codes, got_sb, got_S, w.size), w)
    # byte 0 by hand: element 0 in bits 3..0, element 1 in bits 7..4
    assert got_codes[0] == (codes[0, 0] | (codes[0, 1] << 4))


def test_block_maximum_takes_the_largest_level():
    """With the block scale a normal E4M3 value the block's largest |w| lands within 1/16 of 6, which rounds
    to 6: each block's maximum takes magnitude code 7."""
    W = weights(16, 256, 5)
    codes, sb, S = F.nvfp4_quantize(W)
    c = F.nvfp4_unpack(codes).reshape(-1, 16)
    blocks = W.reshape(-1, 16)
    arg = np.argmax(np.abs(blocks), axis=1)
    normal = sb >= 0x08
    assert normal.mean() > 0.99
    assert np.all((c[np.arange(c.shape[0]), arg] & 7)[normal] == 7)


def test_per_element_error_bound():
    """|w' - w| <= half the gap between the two levels around |n|, times D, plus the roundings of n and w';
    beyond 6 the saturation error |n| - 6 times D."""
    W = weights(32, 512, 6).reshape(-1)
    codes, sb, S = F.nvfp4_quantize(W)
    back = F.nvfp4_dequantize(codes, sb, S, W.size).astype(np.float64)
    Dv = np.repeat(F.nvfp4_block_scales(sb, S), 16).astype(np.float64)
    n = np.abs(W.astype(np.float64)) / Dv
    mags = F.e2m1_table()[:8]
    i = np.clip(np.searchsorted(mags, n), 1, 7)
    half_gap = (mags[i] - mags[i - 1]) / 2
    bound = np.where(n > 6, (n - 6) * Dv, half_gap * Dv) + 4 * np.spacing(np.abs(W)).astype(np.float64) \
        + np.spacing(np.abs(back).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(back - W) <= bound)
    # relative rms error of the order of NF4's on normal weights
    assert 0.05 < np.sqrt(np.mean((back - W) ** 2) / np.mean(W.astype(np.float64) ** 2)) < 0.15


def test_power_of_two_scaling_is_exact():
    W = weights(8, 256, 7).reshape(-1)
    c0, s0, S0 = F.nvfp4_quantize(W)
    c1, s1, S1 = F.nvfp4_quantize((W * np.float32(2.0 ** -6)).astype(np.float32))
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and S1 == S0 * np.float32(2.0 ** -6)


def test_zero_tensor_and_zero_block():
    z = np.zeros(64, np.float32)
    codes, sb, S = F.nvfp4_quantize(z)
    assert S == 0 and not np.any(sb) and not np.any(codes)
    assert not np.any(F.nvfp4_dequantize(codes, sb, S, 64))
    W = weights(1, 64, 8).reshape(-1)
    W[16:32] = 0.0
    codes, sb, S = F.nvfp4_quantize(W)
    assert sb[1] == 0 and not np.any(F.nvfp4_unpack(codes)[16:32])


def test_group_size_from_one_outlier():
    """One large weight in the first block: with groups of 16 the second block keeps its own scale, so its
    largest weight still takes the level 6.  Groups of 32 would put it under the outlier's scale."""
    W = weights(1, 64, 9).reshape(-1)
    W[2] = 1.0
    codes, sb, S = F.nvfp4_quantize(W)
    c = F.nvfp4_unpack(codes)
    assert (c[2] & 7) == 7
    assert np.max(c[16:32] & 7) == 7


@pytest.mark.parametrize("mistake", ["no_tensor_scale", "nibbles_swapped", "ties_away"])
def test_planted_mistakes_are_caught(mistake):
    """Mistakes planted in a copy of the quantizer (on the CPU) break an invariant that the oracle keeps."""
    if mistake == "no_tensor_scale":
        # without S the block scales of small weights (std 0.003) fall among E4M3's coarsest subnormals or to
        # zero: the error is several times that of the two-level scaling
        W = weights(8, 256, 11, std=0.003).reshape(-1)
        blocks = W.reshape(-1, 16)
        t = (np.max(np.abs(blocks), axis=1).astype(np.float64) / 6.0).astype(np.float32)
        sb = F.e4m3_code_of_nonneg(t)
        Dv = F.nvfp4_block_scales(sb, 1.0)
        n = np.where(Dv[:, None] > 0, blocks / np.where(Dv > 0, Dv, 1)[:, None], 0).astype(np.float32)
        back = (F.e2m1_table()[F.e2m1_code_of(n)] * Dv[:, None]).reshape(-1)
        good = F.nvfp4_dequantize(*F.nvfp4_quantize(W), W.size)
        assert np.sqrt(np.mean((back - W) ** 2)) > 3 * np.sqrt(np.mean((good - W) ** 2))
    elif mistake == "nibbles_swapped":
        W = weights(2, 64, 12).reshape(-1)
        codes, sb, S = F.nvfp4_quantize(W)
        swapped = ((codes >> 4) | (codes << 4)).astype(np.uint8)
        assert not np.array_equal(F.nvfp4_dequantize(swapped, sb, S, W.size),
                                  F.nvfp4_dequantize(codes, sb, S, W.size))
    else:
        n = np.array([2.5, 5.0, 0.25], np.float32)
        away = np.array([3.0, 6.0, 0.5])  # ties away from zero
        assert not np.array_equal(F.e2m1_table()[F.e2m1_code_of(n)], away)


# ------------------------------------------------------------------ the FP4 tensor-core form (R24)


def grid_tensor(rows, cols, seed):
    """A tensor on the NVFP4 grid (as in test_worked_tensor_round_trips_exactly): each block holds a +-6 and has a
    normal E4M3 scale, one block reaches 448, so S = 2^-10 and q is the identity."""
    rng = np.random.default_rng(seed)
    nblk = rows * cols // 16
    sb = rng.integers(0x08, 0x7E, nblk).astype(np.uint8)
    sb[0] = 0x7E
    codes = rng.integers(0, 16, (nblk, 16)).astype(np.uint8)
    codes[:, 5] = 0x7
    codes[codes == 0x8] = 0x0
    sval = np.array([D.e4m3_value(int(c)) for c in sb])
    return (F.e2m1_table()[codes] * (sval * 2.0 ** -10)[:, None]).astype(np.float32).reshape(rows, cols)


def test_fp4_forward_on_grid_operands_is_the_plain_product():
    x, W = grid_tensor(4, 64, 1), grid_tensor(6, 64, 2)
    assert np.array_equal(F.nvfp4_roundtrip(x), x) and np.array_equal(F.nvfp4_roundtrip(W), W)
    y = F.fp4_linear_forward(x, W, None, None, 2.0)
    assert np.array_equal(y, x.astype(np.float64) @ W.astype(np.float64).T)


def test_fp4_forward_lora_branch_uses_unquantized_activations():
    """B = 0 leaves the quantized base product; the LoRA term is s (x A^T) B^T with the original x."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((5, 64))).astype(np.float32)
    W = (rng.standard_normal((7, 64)) * 0.02).astype(np.float32)
    A = rng.standard_normal((2, 64)).astype(np.float32)
    B = rng.standard_normal((7, 2)).astype(np.float32)
    base = F.fp4_linear_forward(x, W, None, None, 2.0)
    assert np.array_equal(F.fp4_linear_forward(x, W, A, np.zeros_like(B), 2.0), base)
    lora = F.fp4_linear_forward(x, W, A, B, 2.0) - base
    ref = 2.0 * (x.astype(np.float64) @ A.T.astype(np.float64)) @ B.T.astype(np.float64)
    assert np.allclose(lora, ref, rtol=1e-12, atol=1e-12)
    # and it is not the quantized activations' product
    xq = F.nvfp4_roundtrip(x).astype(np.float64)
    assert not np.allclose(lora, 2.0 * (xq @ A.T.astype(np.float64)) @ B.T.astype(np.float64), rtol=1e-6)


def test_fp4_forward_error_against_the_unquantized_product():
    """On normal operands the FP4 form stays within the sum of the two operands' quantization errors: its
    relative Frobenius distance from x W^T is of the order of sqrt(2) times NVFP4's relative rms error."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    W = (rng.standard_normal((96, 512)) * 0.015).astype(np.float32)
    y = F.fp4_linear_forward(x, W, None, None, 1.0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 0.05 < rel < 0.2
