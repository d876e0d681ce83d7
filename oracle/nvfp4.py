"""NVFP4 base-weight format (quantize / dequantize) -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
------------------
"Major Unsloth Update: NVFP4 Quantization Export and DeepSeek-V4 Training Support" (kongchang.com), section
"NVFP4: A Quantization Format for the Next Generation of Hardware":
- each weight is a 4-bit float in E2M1 encoding (a sign bit, two exponent bits, one mantissa bit), whose
  representable range is about +-6;
- every group of 16 or 32 weights shares one FP8 scaling factor;
- Blackwell's FP4 tensor cores multiply the format directly.

Readings (the pages leave these open)
-------------------------------------
R20 the E2M1 value set: exponent bias 1, a subnormal at exponent field 0, no infinities or NaNs, so the
    magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  A value is rounded to the nearest of them, a tie going to the
    even mantissa bit, and anything beyond 6 in magnitude saturates to +-6; the sign bit is the sign of the
    value being rounded (a negative value that rounds to zero is -0).  This is round-to-nearest-even with
    saturation, the rounding of the hardware's fp32 -> e2m1 conversion.
R21 the group is 16 consecutive weights along a row (the block size of the tensor core's NVFP4 mode); its
    scale is an E4M3 value (OCP FP8, as for the double-quantized constants), rounded to nearest, ties to even.
R22 a second, per-tensor fp32 scale S puts the block scales into the E4M3 range (NVIDIA's two-level NVFP4
    recipe; the pages name only the group scale): S = fl32(amax / 2688), with 2688 = 6 * 448 the product of
    the two formats' largest values, and S = 0 for an all-zero tensor.  For a block with largest magnitude a:
        t = fl32(a / fl32(6 S)),  sb = E4M3 code of t (rounded to nearest even),
        D = fl32(value(sb) * S)           the decoded block scale,
        n = fl32(w / D)                    (n = +0 when D = 0),  code = E2M1 code of n (R20).
    Dequantize: w' = fl32(value(code) * D).
R23 packing: element 2j of the flat row-major weight sits in the LOW nibble of byte j, element 2j + 1 in the
    high nibble -- the order in which the FP4 tensor-core operands are read from memory (the opposite of the
    NF4 packing, reading R5, which the pages leave equally open).

Storage: 0.5 byte per weight for the codes plus 1 byte per 16 weights for the scales (0.5625 byte per weight,
the same as NF4 with fp32 absmax per 64) plus one fp32 per tensor.

R24 (the FP4 tensor-core form of the layer, ``fp4_linear_forward``): see the section at the end.

Pins: ``tests/test_oracle_nvfp4.py``.
"""

from __future__ import annotations

import numpy as np

from .double_quant import e4m3_value

BLOCK = 16            # R21
E2M1_MAX = 6.0        # largest E2M1 magnitude
E4M3_MAX = 448.0
GLOBAL_DIV = E2M1_MAX * E4M3_MAX  # 2688 (R22)


# --------------------------------------------------------------------------------------------------
# E2M1 (R20)
# --------------------------------------------------------------------------------------------------


def e2m1_value(code: int) -> float:
    """Real value of a 4-bit E2M1 pattern: bit 3 sign, bits 2..1 exponent field e (bias 1), bit 0 mantissa m.

    e = 0 is subnormal, m * 0.5; otherwise (1 + m / 2) * 2^(e - 1).
    """
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return sign * m * 0.5
    return sign * (1.0 + m / 2.0) * 2.0 ** (e - 1)


def e2m1_table() -> np.ndarray:
    """fp64 value of each of the 16 codes."""
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def _rne_code(mag: np.ndarray, table_mag: np.ndarray) -> np.ndarray:
    """Index into ascending non-negative magnitudes (index = code, so its low bit is the mantissa bit) of the
    nearest magnitude, ties to the even index; values past the last magnitude take the last."""
    idx = np.searchsorted(table_mag, mag, side="left")  # first magnitude >= mag
    idx = np.clip(idx, 1, table_mag.size - 1)
    lo, hi = table_mag[idx - 1], table_mag[idx]
    below = mag - lo
    above = hi - mag
    pick_hi = (above < below) | ((above == below) & (idx % 2 == 0))
    out = np.where(pick_hi, idx, idx - 1)
    out = np.where(mag >= table_mag[-1], table_mag.size - 1, out)
    out = np.where(mag <= table_mag[0], 0, out)
    return out.astype(np.uint8)


def e2m1_code_of(n: np.ndarray) -> np.ndarray:
    """E2M1 code of fp32 values n: nearest magnitude, ties to even, saturating at 6; the sign bit of n kept."""
    n = np.asarray(n, dtype=np.float32)
    mags = e2m1_table()[:8]  # codes 0..7 ascending: 0, .5, 1, 1.5, 2, 3, 4, 6
    code = _rne_code(np.abs(n).astype(np.float64), mags)
    sign = np.signbit(n).astype(np.uint8) << 3
    return (code | sign).astype(np.uint8)


def e4m3_code_of_nonneg(t: np.ndarray) -> np.ndarray:
    """E4M3 code of non-negative fp32 values: nearest finite value, ties to even, saturating at 448."""
    mags = np.array([e4m3_value(c) for c in range(0x7F)], dtype=np.float64)  # codes 0..0x7E ascending
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    if np.any(t < 0) or np.any(~np.isfinite(t)):
        raise ValueError("block scales are finite and non-negative")
    return _rne_code(t, mags)


# --------------------------------------------------------------------------------------------------
# Quantize / dequantize (R21-R23)
# --------------------------------------------------------------------------------------------------


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def nvfp4_quantize(w: np.ndarray, block: int = BLOCK):
    """NVFP4 quantization of a flat (row-major) fp32 weight.

    Returns ``(codes, scales, S)``: codes uint8 [numel / 2] packed per R23, scales uint8 [numel / block]
    (E4M3 codes), S the fp32 per-tensor scale.
    """
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float32).reshape(-1))
    if w.size % block or w.size % 2 or not np.all(np.isfinite(w)):
        raise ValueError("numel must be a multiple of the block and the weights finite")
    blocks = w.reshape(-1, block)
    amax = np.float32(np.max(np.abs(w))) if w.size else np.float32(0.0)
    S = _f32(np.float64(amax) / GLOBAL_DIV)            # fl32(amax / 2688)
    a = np.max(np.abs(blocks), axis=1)                  # exact
    if S > 0:
        six_s = _f32(6.0 * np.float64(S))               # fl32(6 S)
        t = _f32(a.astype(np.float64) / np.float64(six_s))
    else:
        t = np.zeros(a.shape, dtype=np.float32)
    sb = e4m3_code_of_nonneg(t)
    sv = np.array([e4m3_value(int(c)) for c in range(256)], dtype=np.float64)
    D = _f32(sv[sb] * np.float64(S))                    # fl32(value(sb) * S): exact product, one rounding
    denom = np.where(D > 0, D, np.float32(1.0)).astype(np.float64)
    n = _f32(blocks.astype(np.float64) / denom[:, None])  # the IEEE fp32 quotient
    n = np.where((D > 0)[:, None], n, np.float32(0.0)).astype(np.float32)  # a zero scale gives +0 codes
    code = e2m1_code_of(n).reshape(-1)
    packed = (code[0::2] | (code[1::2] << 4)).astype(np.uint8)  # R23: element 2j in the low nibble
    return packed, sb, S


def nvfp4_unpack(codes: np.ndarray) -> np.ndarray:
    """Packed bytes -> one 4-bit code per element (R23: low nibble first)."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(codes.size * 2, dtype=np.uint8)
    out[0::2] = codes & 0x0F
    out[1::2] = codes >> 4
    return out


def nvfp4_block_scales(scales: np.ndarray, S) -> np.ndarray:
    """Decoded block scales D = fl32(value(sb) * S), fp32 [numel / block]."""
    sv = np.array([e4m3_value(int(c)) for c in range(256)], dtype=np.float64)
    sb = np.asarray(scales, dtype=np.uint8).reshape(-1)
    if np.any(np.isnan(sv[sb])):
        raise ValueError("NaN block scale")
    return _f32(sv[sb] * np.float64(np.float32(S)))


def nvfp4_dequantize(codes: np.ndarray, scales: np.ndarray, S, numel: int, block: int = BLOCK) -> np.ndarray:
    """w' = fl32(value(code) * D_b), fp32 [numel] (the product is exact in fp64 and rounded once)."""
    v = e2m1_table()[nvfp4_unpack(codes)[:numel]]
    D = np.repeat(nvfp4_block_scales(scales, S), block)[:numel]
    return _f32(v * D.astype(np.float64))


# --------------------------------------------------------------------------------------------------
# The FP4 tensor-core form of the layer (R24)
# --------------------------------------------------------------------------------------------------
#
# R24 the block-scaled FP4 MMA multiplies two E2M1 operands, so in that form the activations entering the base
#     product are NVFP4-quantized too, by the same rule as the weight (R20-R22, blocks of 16 along K, their own
#     tensor scale).  The LoRA branch keeps the unquantized activations (the adapters are trained in bf16).
#         y = q(x) q(W)^T + s (x A^T) B^T,   q = NVFP4 quantize-then-dequantize,
#     in fp64 from the dequantized fp32 operands.


def nvfp4_roundtrip(a: np.ndarray) -> np.ndarray:
    """q(a): the fp32 values a [rows, K] takes after NVFP4 quantization and dequantization (K % 16 == 0)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    codes, scales, S = nvfp4_quantize(a.reshape(-1))
    return nvfp4_dequantize(codes, scales, S, a.size).reshape(a.shape)


def fp4_linear_forward(x, W, A, B, s: float) -> np.ndarray:
    """y [M, N] in fp64 for the FP4 tensor-core form (R24): x [M, K] (bf16 values), W [N, K] fp32."""
    xq = nvfp4_roundtrip(x).astype(np.float64)
    wq = nvfp4_roundtrip(W).astype(np.float64)
    x64 = np.asarray(x, dtype=np.float64)
    y = xq @ wq.T
    if A is not None and np.asarray(A).shape[0] > 0:
        y = y + float(s) * ((x64 @ np.asarray(A, dtype=np.float64).T) @ np.asarray(B, dtype=np.float64).T)
    return y
