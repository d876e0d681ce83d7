"""LoRA merge and NF4 requantization oracle -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
------------------
"unsloth" (pyshine.com), section "Why You Need This", the paragraph on saving: a fine-tuned model is saved
either as its adapters or merged, with the LoRA weights folded into the base layer by layer.  The merged
weight of one layer is W' = deq(W) + s B A  ([N,K]; A [r,K], B [N,r], s the LoRA scaling).

Readings (the pages are silent on each)
---------------------------------------
R15  precision and order.  Every step is one IEEE fp32 operation, in this order, with no fused multiply-add:
         d    = fl32(level[code] * absmax)                      the dequantized base (as nf4_dequantize)
         p_j  = fl32(B[n,j] * A[j,k])                           exact: a product of two bf16 values fits fp32
         acc  = (((p_0 + p_1) + p_2) + ...) + p_{r-1}            left to right in fp32; acc = 0 when r = 0
         w'   = fl32(d + fl32(s * acc))
     A summation order has to be fixed because the merged weight is requantized, and a quantization
     decision must be taken on the same fp32 value on both sides.
R16  requantization.  The merged weight is quantized by the same blockwise NF4 rule as the base weight
     (``oracle.nf4.nf4_quantize``), so the merged model stays in 4-bit; the bf16 output is w' rounded to
     nearest-even.

Pins: ``tests/test_oracle_merge.py`` (B = 0 and s = 0 give back the base exactly, and quantize(dequantize)
is the identity on codes and scales; a hand-expanded single-column case; the recursive-summation error bound
against the fp64 product; the nearest-level property of the requantized codes).
"""

from __future__ import annotations

import numpy as np

from . import nf4 as O


def merge_lora(codes: np.ndarray, absmax: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, N: int,
               K: int) -> np.ndarray:
    """W' [N,K] fp32 by R15.  A [r,K] and B [N,r] hold bf16 values (given as float arrays)."""
    d = O.nf4_dequantize(codes, absmax, N * K).reshape(N, K).astype(np.float32)
    A32 = np.asarray(A, dtype=np.float32)
    B32 = np.asarray(B, dtype=np.float32)
    r = A32.shape[0] if A32.ndim == 2 else 0
    acc = np.zeros((N, K), dtype=np.float32)
    for j in range(r):
        # fp32 products (exact for bf16 operands), added to the running sum one rank at a time
        acc = acc + np.outer(B32[:, j], A32[j, :]).astype(np.float32)
    t = (np.float32(s) * acc).astype(np.float32)
    return (d + t).astype(np.float32)


def merge_lora_bf16_bits(codes, absmax, A, B, s, N, K) -> np.ndarray:
    """W' rounded to bf16 (R16), as uint16 bit patterns [N,K]."""
    return O.f32_to_bf16_bits(merge_lora(codes, absmax, A, B, s, N, K))


def merge_lora_nf4(codes, absmax, A, B, s, N, K):
    """(codes', absmax'): W' requantized by the blockwise NF4 rule (R16)."""
    return O.nf4_quantize(merge_lora(codes, absmax, A, B, s, N, K).ravel())
