"""Double quantization of the NF4 block constants -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
------------------
"Unsloth v0.1.463-beta: Fixes Studio Crash and llama-server Permission Issue" (kongchang.com), section
"About the Unsloth Project", paragraph "How LoRA and QLoRA work": beside the 4-bit NF4 base weight, QLoRA
quantizes the quantization constants themselves a second time ("double quantization"), which is part of how
it brings the memory of fine-tuning a 65B model down to about 48 GB.  The pages give neither the second
format, nor its block size, nor the centring.  The readings below fill those in.

Readings (the pages are silent on each)
---------------------------------------
R17 the constants are the fp32 absmax values of the 64-element NF4 blocks, in flat (row-major) order.  They
    are quantized again in groups of 256 consecutive constants (the last group may be shorter), after
    subtracting one offset for the whole tensor, mu = their mean (the constants are all >= 0; centring lets
    a symmetric 8-bit format cover them).  Each group keeps one fp32 scale c1 = max |d| over the group,
    d = fl32(absmax - mu); each constant keeps an 8-bit code for n = fl32(d / c1) (n = 0 when c1 = 0).
    This is the rule of the QLoRA method (8-bit float codes, 256 constants per group, mean subtracted).
R18 the 8-bit float is OCP FP8 E4M3 (bias 7, no infinities, 0x7F / 0xFF are NaN, largest finite 448), the
    8-bit float format sm_100 converts and multiplies natively.  Its finite values divided by 448, each
    rounded once to fp32, are the level set L; a code is the E4M3 bit pattern of its level (0 -> 0x00).
    n takes the nearest level, a value exactly between two levels the lower one (as NF4's R2).
R19 the mean is computed in a fixed order so that it is one number: each group's constants summed in fp64
    in index order, the group sums added in fp64 in group order, the total divided by the count in fp64,
    rounded once to fp32.
Dequantize: absmax' = fl32(fl32(L[code] * c1) + mu): an fp32 product, then an fp32 sum.

Storage: 1 byte per 64 weights plus 4 bytes per 256 x 64 weights, about 0.127 bit per weight instead of 0.5.

Pins: ``tests/test_oracle_double_quant.py`` (the E4M3 decoding against torch's float8 type, nearest-level
codes by brute force, the offset against an exactly rounded sum, the group size through the count of
extreme codes, error bounds, constant and scaled inputs, planted mistakes).
"""

from __future__ import annotations

import numpy as np

GROUP = 256        # constants per second-level group (R17)
E4M3_MAX = 448.0   # largest finite E4M3 value (R18)


# --------------------------------------------------------------------------------------------------
# The E4M3 level set (R18)
# --------------------------------------------------------------------------------------------------


def e4m3_value(code: int) -> float:
    """The real value of an E4M3 bit pattern (NaN for 0x7F / 0xFF), from the format's definition.

    Bit 7 is the sign, bits 6..3 the exponent field e (bias 7), bits 2..0 the mantissa field m.  e = 0 is
    subnormal, m / 8 * 2^-6; otherwise (1 + m / 8) * 2^(e - 7).  The all-ones exponent with m = 7 is NaN;
    the format has no infinities, so e = 15 with m < 7 are ordinary values (up to 1.75 * 2^8 = 448).
    """
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """fp64 value of each of the 256 codes (NaN at 0x7F and 0xFF)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def dq_levels() -> np.ndarray:
    """L[code] = fl32(value(code) / 448) for every code, fp32 [256] (NaN codes stay NaN)."""
    return (e4m3_table() / E4M3_MAX).astype(np.float32)


def dq_sorted_levels() -> tuple[np.ndarray, np.ndarray]:
    """The distinct levels in ascending order and the code each one is stored as.

    -0 (0x80) repeats +0 and is never produced; the two NaN codes are not levels.  253 levels remain.
    """
    lev = dq_levels()
    codes = [c for c in range(256) if c not in (0x7F, 0xFF, 0x80)]
    codes.sort(key=lambda c: float(lev[c]))
    codes = np.array(codes, dtype=np.uint8)
    return lev[codes], codes


def dq_code_of(n: np.ndarray) -> np.ndarray:
    """Code of normalised fp32 values n (|n| <= 1): the nearest level, a tie going to the lower one (R18).

    The index into the ascending levels is the number of midpoints strictly below n; each midpoint of two
    fp32 levels is exact in fp64.
    """
    vals, codes = dq_sorted_levels()
    v = vals.astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2.0
    n64 = np.asarray(n, dtype=np.float32).astype(np.float64)
    idx = np.searchsorted(mids, n64, side="left")  # count of midpoints < n
    return codes[idx]


# --------------------------------------------------------------------------------------------------
# Offset, quantize, dequantize
# --------------------------------------------------------------------------------------------------


def dq_offset(absmax: np.ndarray, group: int = GROUP) -> np.float32:
    """mu per R19: fp64 sums group by group in index order, then over the groups in order, / count, -> fp32."""
    c = np.asarray(absmax, dtype=np.float32).reshape(-1).astype(np.float64).tolist()  # Python floats are fp64
    if not c:
        return np.float32(0.0)
    total = 0.0
    for g0 in range(0, len(c), group):
        part = 0.0
        for v in c[g0:g0 + group]:  # in index order
            part += v
        total += part
    return np.float32(total / float(len(c)))


def dq_quantize(absmax: np.ndarray, group: int = GROUP):
    """Double-quantize the flat fp32 block constants (R17-R19).

    Returns ``(code8, c1, mu)``: code8 uint8 [nb], c1 fp32 [ceil(nb / group)], mu an fp32 scalar.
    """
    c = np.ascontiguousarray(np.asarray(absmax, dtype=np.float32).reshape(-1))
    if not np.all(np.isfinite(c)) or np.any(c < 0):
        raise ValueError("block constants must be finite and non-negative")
    nb = c.size
    mu = dq_offset(c, group)
    # d = fl32(c - mu): the fp64 difference of two fp32 values rounded once to fp32 is the fp32 difference
    d = (c.astype(np.float64) - np.float64(mu)).astype(np.float32)
    ng = (nb + group - 1) // group
    c1 = np.zeros(ng, dtype=np.float32)
    code8 = np.zeros(nb, dtype=np.uint8)
    for g in range(ng):
        dg = d[g * group:(g + 1) * group]
        c1[g] = np.max(np.abs(dg)) if dg.size else np.float32(0.0)
        if c1[g] > 0:
            n = (dg.astype(np.float64) / np.float64(c1[g])).astype(np.float32)  # the IEEE fp32 quotient
        else:
            n = np.zeros(dg.shape, dtype=np.float32)
        code8[g * group:(g + 1) * group] = dq_code_of(n)
    return code8, c1, mu


def dq_dequantize(code8: np.ndarray, c1: np.ndarray, mu, group: int = GROUP) -> np.ndarray:
    """absmax' = fl32(fl32(L[code] * c1_g) + mu), fp32 [nb]."""
    code8 = np.asarray(code8, dtype=np.uint8).reshape(-1)
    lev = dq_levels()
    if np.any(np.isnan(lev[code8])):
        raise ValueError("NaN code in the double-quantized constants")
    scale = np.repeat(np.asarray(c1, dtype=np.float32), group)[:code8.size]
    prod = (lev[code8].astype(np.float64) * scale.astype(np.float64)).astype(np.float32)  # exact, rounded once
    return (prod.astype(np.float64) + np.float64(np.float32(mu))).astype(np.float32)


def nf4_dequantize_dq(codes, code8, c1, mu, numel: int, blocksize: int = 64, group: int = GROUP) -> np.ndarray:
    """The NF4 weight with double-quantized constants: NF4 dequantization with absmax' in place of absmax."""
    from . import nf4
    return nf4.nf4_dequantize(codes, dq_dequantize(code8, c1, mu, group), numel, blocksize)
