"""QLoRA linear layer oracle (fp64) -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix
------------------
"Unsloth v0.1.463-beta: Fixes Studio Crash and llama-server Permission Issue" (kongchang.com), section
"About the Unsloth Project", paragraph "How LoRA and QLoRA work": the weight update is the low-rank product
dW = B A of rank r; only A and B are trained; the base weight is frozen in NF4.
"unsloth" (pyshine.com), section "Why You Need This": one call computes the base product with the
quantized weight and the adapter delta together.  "Inside Unsloth: How the Fastest LLM Fine-Tuning
Library Works" (thriftbooks.com), section "What You'll Learn", item "LoRA and QLoRA": NF4 dequantization,
the matrix multiplication and the LoRA correction are one launch.

Definitions written out (all arithmetic fp64 on the given inputs; matmul is a library primitive):
    forward   y  = x Wd^T + s (x A^T) B^T
    backward  dX = dY Wd + s (dY B) A
              dA = s (dY B)^T x
              dB = s dY^T (x A^T)
with x [M,K], Wd [N,K] the dequantized base weight, A [r,K], B [N,r], dY [M,N].  W is frozen: no dW.

Readings: R7 -- the scaling s is lora_alpha / r ("unsloth" (pyshine.com), section "From Install to a
Fine-Tuned Model", the ``r`` and ``lora_alpha`` arguments); the layer takes s itself.  R8 -- dY is an
external input.  R10 -- in the gated-MLP chain the gate/up outputs and the SwiGLU output are stored as
bf16 between the layers, as a fine-tuning framework stores activations; ``mlp_chain_*`` applies those
roundings by default and skips them with ``round_intermediates=False``.

SwiGLU ("Inside Unsloth ...", section "What You'll Learn", item "Triton Kernel Internals"; "unsloth"
(pyshine.com), the kernels-directory paragraph naming swiglu.py):
    silu(g) = g / (1 + exp(-g)),   h = silu(g) * up
    dg  = dh * up * sigma(g) * (1 + g (1 - sigma(g))),   dup = dh * silu(g)

Pins: ``tests/test_oracle_linear.py``.
"""

from __future__ import annotations

import numpy as np

from .nf4 import nf4_dequantize, round_bf16


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def dequantized_weight(codes, absmax, N: int, K: int, blocksize: int = 64) -> np.ndarray:
    """Wd [N,K] in fp64: the fp32 dequantized weight w' (exact values) widened to fp64."""
    return nf4_dequantize(codes, absmax, N * K, blocksize).astype(np.float64).reshape(N, K)


# --------------------------------------------------------------------------------------------------
# The linear layer
# --------------------------------------------------------------------------------------------------


def lora_down(x, A) -> np.ndarray:
    """u = x A^T  [M,r]."""
    return _f64(x) @ _f64(A).T


def qlora_forward(x, Wd, A, B, s: float) -> np.ndarray:
    """y = x Wd^T + s (x A^T) B^T  [M,N]."""
    x = _f64(x)
    return x @ _f64(Wd).T + float(s) * (lora_down(x, A) @ _f64(B).T)


def lora_grads(dy, x, A, B, s: float):
    """(dA [r,K], dB [N,r]): the adapter gradients, which do not involve the base weight."""
    dy, x, A, B = _f64(dy), _f64(x), _f64(A), _f64(B)
    s = float(s)
    v = dy @ B                      # dY B   [M,r]
    dA = s * (v.T @ x)
    dB = s * (dy.T @ (x @ A.T))
    return dA, dB


def qlora_backward(dy, x, Wd, A, B, s: float):
    """(dX [M,K], dA [r,K], dB [N,r]) of the forward above, for the upstream gradient dY [M,N]."""
    dy, x, Wd, A, B = _f64(dy), _f64(x), _f64(Wd), _f64(A), _f64(B)
    s = float(s)
    dx = dy @ Wd + s * ((dy @ B) @ A)
    dA, dB = lora_grads(dy, x, A, B, s)
    return dx, dA, dB


# --------------------------------------------------------------------------------------------------
# SwiGLU
# --------------------------------------------------------------------------------------------------


def sigmoid(g) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-_f64(g)))


def silu(g) -> np.ndarray:
    g = _f64(g)
    return g / (1.0 + np.exp(-g))


def silu_grad(g) -> np.ndarray:
    """d silu / dg = sigma(g) (1 + g (1 - sigma(g)))."""
    g = _f64(g)
    sg = sigmoid(g)
    return sg * (1.0 + g * (1.0 - sg))


def swiglu_forward(g, up) -> np.ndarray:
    return silu(g) * _f64(up)


def swiglu_backward(dh, g, up):
    """(dg, dup) for h = silu(g) * up."""
    dh, g, up = _f64(dh), _f64(g), _f64(up)
    return dh * up * silu_grad(g), dh * silu(g)


# --------------------------------------------------------------------------------------------------
# Gated MLP chain: gate/up projections, SwiGLU, down projection (each projection a QLoRA linear)
# --------------------------------------------------------------------------------------------------


def _bf16(a) -> np.ndarray:
    return round_bf16(np.asarray(a, dtype=np.float32)).astype(np.float64)


def mlp_chain_forward(x, gate, up, down, round_intermediates: bool = True):
    """Forward of the chain.  ``gate``/``up``/``down`` are (Wd, A, B, s) tuples.

    Returns (y, g, u, h): with ``round_intermediates`` the stored activations g, u, h are bf16 (R10).
    """
    rnd = _bf16 if round_intermediates else _f64
    g = rnd(qlora_forward(x, *gate))
    u = rnd(qlora_forward(x, *up))
    h = rnd(swiglu_forward(g, u))
    y = qlora_forward(h, *down)
    return y, g, u, h


def mlp_chain_backward(dy, x, gate, up, down, saved, round_intermediates: bool = True):
    """Backward of the chain given the forward's (g, u, h).  Returns dX and the (dA, dB) of each layer.

    With ``round_intermediates`` the gradients that cross a layer boundary (dh, dg, dup) are bf16 (R10).
    """
    rnd = _bf16 if round_intermediates else _f64
    g, u, h = saved
    dh, dA_down, dB_down = qlora_backward(dy, h, *down)
    dh = rnd(dh)
    dg, du = swiglu_backward(dh, g, u)
    dg, du = rnd(dg), rnd(du)
    dx_g, dA_gate, dB_gate = qlora_backward(dg, x, *gate)
    dx_u, dA_up, dB_up = qlora_backward(du, x, *up)
    return dx_g + dx_u, {"gate": (dA_gate, dB_gate), "up": (dA_up, dB_up), "down": (dA_down, dB_down)}


# --------------------------------------------------------------------------------------------------
# Tolerance used to compare a GPU result with the fp64 oracle
# --------------------------------------------------------------------------------------------------

REL_FRO_TOL = 1e-2
MAX_ABS_TOL_FRAC = 2e-2


def compare(got, ref) -> dict:
    """Relative Frobenius error and max-abs error (as a fraction of max |ref|) of ``got`` against ``ref``."""
    got, ref = _f64(got), _f64(ref)
    diff = got - ref
    ref_norm = float(np.linalg.norm(ref))
    ref_max = float(np.max(np.abs(ref))) if ref.size else 0.0
    rel_fro = float(np.linalg.norm(diff)) / ref_norm if ref_norm > 0 else float(np.linalg.norm(diff))
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    max_frac = max_abs / ref_max if ref_max > 0 else max_abs
    ok = rel_fro <= REL_FRO_TOL and max_frac <= MAX_ABS_TOL_FRAC
    return {"rel_fro": rel_fro, "max_abs_frac": max_frac, "ok": ok}
