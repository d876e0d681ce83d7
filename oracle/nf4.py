"""NF4 blockwise quantization oracle -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
------------------
"Unsloth v0.1.463-beta: Fixes Studio Crash and llama-server Permission Issue" (kongchang.com), section
"About the Unsloth Project", paragraph "How LoRA and QLoRA work": the frozen base weight is stored as 4-bit
NormalFloat (NF4) codes, a level set designed for normally distributed weights, with quantization
constants kept beside the codes; the LoRA adapters stay in bf16.  "unsloth" (pyshine.com), section "Why You
Need This": NF4 weights are dequantized on the fly.  No page prints the level table, the block size, the
rounding rule or the packing, so the readings below fill those in.

Readings (the pages are silent on each)
---------------------------------------
R1  level set: the normal-quantile rule of the QLoRA method -- 8 positive and 7 negative quantiles of the
    standard normal at evenly spaced probabilities from 1 - delta down to 1/2 (delta = (1/32 + 1/30)/2),
    normalised by the largest, plus an exact 0; each level rounded once to fp32.
R2  a value exactly on the midpoint of two levels takes the lower code.
R3  an all-zero block stores absmax 0 and every code is the zero level (index 7).
R4  non-finite weights are outside the operation's domain (rejected here).
R5  packing: element 2j of the flat row-major weight sits in the HIGH nibble (bits 7..4) of byte j,
    element 2j+1 in the low nibble.
Quantize:   absmax_b = max |w| over the block (exact in fp32); n = fl32(w / absmax_b) (IEEE fp32 quotient);
            code = number of midpoints m_i = (c_i + c_{i+1})/2 (exact in fp64) strictly below n.
Dequantize: w' = fl32(c[code] * absmax_b); bf16 output = round-to-nearest-even of w'.

Pins: ``tests/test_oracle_nf4.py``.  The pages print no table, so the level set is pinned to the outside
source that defines NF4: the 16 values printed in the QLoRA paper (Dettmers et al., 2023, Appendix E), which
this construction reproduces to within 8 fp32 ulps (relative 7e-7); planted slips in the construction (a
wrong delta, a wrong probability grid, uniform instead of normal quantiles) miss them by orders of
magnitude.  Invariants and a second, independent normal-quantile routine pin the rest.
"""

from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------------------
# Standard-normal quantile, by bisection on the complementary error function (fp64).
# --------------------------------------------------------------------------------------------------


def normal_cdf(z: float) -> float:
    """Phi(z) = erfc(-z / sqrt 2) / 2, in fp64."""
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def normal_quantile(p: float) -> float:
    """Phi^{-1}(p) for 0 < p < 1, by bisection until the bracket is two adjacent doubles.

    Below 1/2 it bisects on Phi(z) = erfc(-z/sqrt 2)/2; above 1/2 on the upper tail
    1 - Phi(z) = erfc(z/sqrt 2)/2 against 1 - p (exact for p >= 1/2), which avoids the cancellation of
    erfc near 2.  Phi^{-1}(1/2) = 0 exactly.
    """
    if not (0.0 < p < 1.0):
        raise ValueError("normal_quantile needs 0 < p < 1")
    if p == 0.5:
        return 0.0
    if p < 0.5:
        target, f, increasing = p, normal_cdf, True
    else:
        target, f, increasing = 1.0 - p, (lambda z: 0.5 * math.erfc(z / math.sqrt(2.0))), False
    lo, hi = -40.0, 40.0
    for _ in range(4000):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        below = f(mid) < target
        if below == increasing:
            lo = mid
        else:
            hi = mid
    return lo if abs(f(lo) - target) <= abs(f(hi) - target) else hi


# --------------------------------------------------------------------------------------------------
# Codebook (reading R1)
# --------------------------------------------------------------------------------------------------

NF4_DELTA = 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def nf4_probabilities() -> tuple[list[float], list[float]]:
    """The probabilities whose quantiles give the positive (8) and negative (7) levels, per R1.

    Positive side: 9 evenly spaced points from 1 - delta down to 1/2, the last (1/2, the zero) dropped.
    Negative side: 8 evenly spaced points over the same range, the last dropped; their quantiles negated.
    """
    top = 1.0 - NF4_DELTA
    pos = [top + i * (0.5 - top) / 8.0 for i in range(8)]
    neg = [top + i * (0.5 - top) / 7.0 for i in range(7)]
    return pos, neg


def nf4_codebook_f64() -> np.ndarray:
    """The 16 levels in fp64 before the fp32 rounding, ascending (R1)."""
    pos, neg = nf4_probabilities()
    qpos = [normal_quantile(p) for p in pos]
    qneg = [-normal_quantile(p) for p in neg]
    scale = max(qpos + [-q for q in qneg])
    levels = [q / scale for q in qpos] + [q / scale for q in qneg] + [0.0]
    return np.array(sorted(levels), dtype=np.float64)


def nf4_codebook() -> np.ndarray:
    """The NF4 codebook: the R1 levels each rounded once to fp32, ascending, c[7] == 0, c[0] == -1, c[15] == 1."""
    return nf4_codebook_f64().astype(np.float32)


def nf4_midpoints(codebook: np.ndarray | None = None) -> np.ndarray:
    """m_i = (c_i + c_{i+1}) / 2 for i = 0..14, exact in fp64 (a sum of two fp32 values and a halving)."""
    c = (nf4_codebook() if codebook is None else codebook).astype(np.float64)
    return (c[:-1] + c[1:]) / 2.0


# --------------------------------------------------------------------------------------------------
# Quantize / dequantize
# --------------------------------------------------------------------------------------------------


def nf4_code_of(n: np.ndarray, codebook: np.ndarray | None = None) -> np.ndarray:
    """Code of already-normalised fp32 values n: how many midpoints lie strictly below n (R2: ties go low)."""
    n64 = np.asarray(n, dtype=np.float32).astype(np.float64)
    mids = nf4_midpoints(codebook)
    code = np.zeros(n64.shape, dtype=np.uint8)
    for m in mids:
        code += (n64 > m).astype(np.uint8)
    return code


def nf4_quantize(w: np.ndarray, blocksize: int = 64, codebook: np.ndarray | None = None):
    """Blockwise NF4 quantization of a flat (row-major) fp32 weight.

    Returns ``(codes, absmax)``: codes uint8 [numel/2] packed per R5, absmax fp32 [numel/blocksize].
    """
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float32).reshape(-1))
    numel = w.size
    if blocksize <= 0 or numel % blocksize != 0 or numel % 2 != 0 or blocksize % 2 != 0:
        raise ValueError("numel must be a multiple of an even blocksize")
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight (outside the operation's domain, reading R4)")
    blocks = w.reshape(-1, blocksize)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)  # exact: a max of fp32 magnitudes
    # n = fl32(w / absmax): the fp64 quotient rounded once to fp32 equals the IEEE fp32 quotient
    # (double rounding through a 53-bit format is harmless for a quotient of two 24-bit numbers).
    denom = np.where(absmax > 0, absmax, np.float32(1.0)).astype(np.float64)
    n = (blocks.astype(np.float64) / denom[:, None]).astype(np.float32)
    n[absmax == 0] = 0.0  # R3
    code = nf4_code_of(n, codebook).reshape(-1)
    packed = ((code[0::2] << 4) | code[1::2]).astype(np.uint8)  # R5
    return packed, absmax


def nf4_unpack(codes: np.ndarray) -> np.ndarray:
    """Packed bytes -> one code per element (R5: high nibble first)."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(codes.size * 2, dtype=np.uint8)
    out[0::2] = codes >> 4
    out[1::2] = codes & 0x0F
    return out


def nf4_dequantize(codes: np.ndarray, absmax: np.ndarray, numel: int, blocksize: int = 64,
                   codebook: np.ndarray | None = None) -> np.ndarray:
    """w' = fl32(c[code] * absmax_b) as fp32 [numel] (the fp32 product computed exactly in fp64, rounded once)."""
    c = nf4_codebook() if codebook is None else np.asarray(codebook, dtype=np.float32)
    idx = nf4_unpack(codes)[:numel]
    scale = np.repeat(np.asarray(absmax, dtype=np.float32), blocksize)[:numel]
    return (c[idx].astype(np.float64) * scale.astype(np.float64)).astype(np.float32)


def nf4_dequantize_bf16_bits(codes, absmax, numel, blocksize=64, codebook=None) -> np.ndarray:
    """bf16 dequantization: round-to-nearest-even of the fp32 w', returned as uint16 bit patterns."""
    return f32_to_bf16_bits(nf4_dequantize(codes, absmax, numel, blocksize, codebook))


# --------------------------------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even), on bit patterns
# --------------------------------------------------------------------------------------------------


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16, ties to even; returns the uint16 bit patterns.

    bf16 keeps the top 16 bits of the fp32 pattern.  Adding 0x7FFF plus the lowest kept bit and truncating
    rounds the dropped 16 bits to nearest, with an exact half going to the even kept pattern.
    """
    b = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    if not np.all(np.isfinite(np.asarray(a, dtype=np.float32))):
        raise ValueError("f32_to_bf16_bits handles finite values only")
    keep_lsb = (b >> 16) & 1
    return ((b + 0x7FFF + keep_lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Values rounded to the nearest bf16 (ties to even), as fp32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(a, dtype=np.float32)))
