"""Seeded synthetic inputs for the QLoRA linear layer workloads.

This module only draws random numbers and rounds them to the storage dtypes; it holds none of the layer's
arithmetic.  Both the GPU tests and the oracle tests take their inputs from here, and so does the
benchmark.  Every draw comes from numpy's PCG64 generator with a stated seed, in a fixed order, so any
machine reproduces the same tensors.

Workloads (the shapes and distributions the layer is measured on):

==========================  =====  =====  =====  ===  ===  =========  ====================================
name                          M      K      N     r    s    W std     x
==========================  =====  =====  =====  ===  ===  =========  ====================================
tiny_64x256x256_r8             64    256    256    8   2    0.02      N(0,1)
attn_2048x4096x4096_r16      2048   4096   4096   16   2    0.02      N(0,1)
mlpdown_4096x11008x4096_r64  4096  11008   4096   64   1    0.02      silu(g)*u, g,u ~ N(0,1) (fp32)
decode_16x8192x28672_r16       16   8192  28672   16   2    0.015     N(0,1)      (forward only)
==========================  =====  =====  =====  ===  ===  =========  ====================================

plus the gated-MLP chain ``mlpchain_8192x8192x28672_r64``: x [8192,8192] ~ N(0,1); gate and up W
[28672,8192], down W [8192,28672], each ~ N(0,0.015^2) with its own seed and its own LoRA pair, r=64, s=2.

Distributions: x ~ N(0,1) rounded to bf16; W ~ N(0, std^2) kept fp32 (it is quantized to NF4 by the
library); A ~ U(-1/sqrt(K), +1/sqrt(K)) rounded to bf16; B ~ N(0, 0.01^2) rounded to bf16; the upstream
gradient dY ~ N(0,1) rounded to bf16 from its own seed (1).  Each tensor has its own PCG64 stream spawned
from ``SeedSequence(seed)`` (seed 0 for a workload): x (or the g of a SwiGLU-shaped x), u, W, A, B.  Streams
fill row-major, so the first M' rows of x drawn for M tokens equal x drawn for M' tokens.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class LinearWorkload:
    name: str
    M: int
    K: int
    N: int
    r: int
    s: float
    w_std: float
    x_kind: str = "normal"      # "normal" | "swiglu"
    backward: bool = True

    @property
    def flops_fwd(self) -> int:
        """2MNK for the base product + 2MKr + 2MNr for the LoRA term."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r

    @property
    def flops_bwd(self) -> int:
        """dX: 2MNK + 2MNr + 2MrK;  dA: 2rMK;  dB: 2NMr."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return (2 * M * N * K + 2 * M * N * r + 2 * M * r * K) + 2 * r * M * K + 2 * N * M * r

    @property
    def bytes_fwd(self) -> int:
        """NF4 weight once (0.5 B codes + 4/64 B absmax per element), x read, y written, A and B read."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return N * K // 2 + N * K // 64 * 4 + 2 * M * K + 2 * M * N + 2 * r * K + 2 * N * r

    @property
    def bytes_bwd(self) -> int:
        """NF4 weight once, dY and x read, dX written, A and B read, dA and dB written (fp32)."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return (N * K // 2 + N * K // 64 * 4 + 2 * M * N + 2 * M * K + 2 * M * K
                + 2 * r * K + 2 * N * r + 4 * r * K + 4 * N * r)


WORKLOADS = {
    w.name: w
    for w in [
        LinearWorkload("tiny_64x256x256_r8", 64, 256, 256, 8, 2.0, 0.02),
        LinearWorkload("attn_2048x4096x4096_r16", 2048, 4096, 4096, 16, 2.0, 0.02),
        LinearWorkload("mlpdown_4096x11008x4096_r64", 4096, 11008, 4096, 64, 1.0, 0.02, x_kind="swiglu"),
        LinearWorkload("decode_16x8192x28672_r16", 16, 8192, 28672, 16, 2.0, 0.015, backward=False),
    ]
}

CHAIN = dict(name="mlpchain_8192x8192x28672_r64", M=8192, D=8192, F=28672, r=64, s=2.0, w_std=0.015)


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy array -> bf16 CPU tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _streams(seed: int) -> list[np.random.Generator]:
    """Five independent streams: x (or g), u, W, A, B."""
    return [np.random.Generator(np.random.PCG64(ss)) for ss in np.random.SeedSequence(seed).spawn(5)]


def draw_x(streams, M: int, K: int, kind: str = "normal") -> torch.Tensor:
    if kind == "normal":
        return to_bf16(streams[0].standard_normal((M, K), dtype=np.float32))
    if kind == "swiglu":
        # activations distributed like the output of a SwiGLU unit fed N(0,1) inputs (fp32, then bf16)
        g = streams[0].standard_normal((M, K), dtype=np.float32)
        u = streams[1].standard_normal((M, K), dtype=np.float32)
        return to_bf16(g / (np.float32(1.0) + np.exp(-g)) * u)
    raise ValueError(kind)


def draw_w(streams, N: int, K: int, std: float) -> np.ndarray:
    return streams[2].standard_normal((N, K), dtype=np.float32) * np.float32(std)


def draw_lora(streams, N: int, K: int, r: int):
    a = np.float32(1.0 / np.sqrt(K))
    A = to_bf16(streams[3].uniform(-a, a, size=(r, K)).astype(np.float32))
    B = to_bf16(streams[4].standard_normal((N, r), dtype=np.float32) * np.float32(0.01))
    return A, B


def draw_dy(M: int, N: int, seed: int = 1) -> torch.Tensor:
    return to_bf16(_rng(seed).standard_normal((M, N), dtype=np.float32))


def make_linear_inputs(w: LinearWorkload | str, seed: int = 0, M: int | None = None):
    """x [M,K] bf16, W [N,K] fp32, A [r,K] bf16, B [N,r] bf16, dY [M,N] bf16 (CPU tensors / arrays).

    ``M`` overrides the token count; x and dY are then the first M rows of the full draws and W, A, B are
    unchanged (used for bounded sub-batches).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    M = w.M if M is None else M
    st = _streams(seed)
    x = draw_x(st, M, w.K, w.x_kind)
    W = draw_w(st, w.N, w.K, w.w_std)
    A, B = draw_lora(st, w.N, w.K, w.r)
    dy = draw_dy(M, w.N, seed + 1)
    return dict(x=x, W=W, A=A, B=B, dy=dy, s=w.s, M=M, N=w.N, K=w.K, r=w.r)


def make_random_linear(M: int, N: int, K: int, r: int, s: float = 2.0, seed: int = 0, w_std: float = 0.02):
    """Same recipe as the workloads for an arbitrary shape (used for ragged / edge-case tests)."""
    st = _streams(seed)
    x = draw_x(st, M, K)
    W = draw_w(st, N, K, w_std)
    A, B = draw_lora(st, N, K, r) if r > 0 else (to_bf16(np.zeros((0, K), np.float32)),
                                                  to_bf16(np.zeros((N, 0), np.float32)))
    dy = draw_dy(M, N, seed + 1)
    return dict(x=x, W=W, A=A, B=B, dy=dy, s=s, M=M, N=N, K=K, r=r)


def make_chain_inputs(M: int | None = None, D: int | None = None, F: int | None = None, r: int | None = None,
                      s: float | None = None, w_std: float | None = None):
    """Gated-MLP chain inputs: x [M,D]; gate/up W [F,D]; down W [D,F]; LoRA (A,B) per layer; dY [M,D].

    Seeds: x 0, dY 1, gate 2, up 3, down 4.
    """
    M = CHAIN["M"] if M is None else M
    D = CHAIN["D"] if D is None else D
    F = CHAIN["F"] if F is None else F
    r = CHAIN["r"] if r is None else r
    s = CHAIN["s"] if s is None else s
    w_std = CHAIN["w_std"] if w_std is None else w_std
    x = draw_x(_streams(0), M, D)
    layers = {}
    for name, seed, (n, k) in (("gate", 2, (F, D)), ("up", 3, (F, D)), ("down", 4, (D, F))):
        st = _streams(seed)
        W = draw_w(st, n, k, w_std)
        A, B = draw_lora(st, n, k, r)
        layers[name] = dict(W=W, A=A, B=B, s=s, N=n, K=k, r=r)
    dy = draw_dy(M, D, 1)
    return dict(x=x, dy=dy, layers=layers, M=M, D=D, F=F, r=r, s=s)


def make_chain_sample(m: int, f: int, D: int | None = None, F: int | None = None, r: int | None = None,
                      s: float | None = None, w_std: float | None = None):
    """A bounded sample of the gated-MLP chain: its first ``m`` tokens and first ``f`` intermediate features.

    Every tensor equals the matching slice of ``make_chain_inputs(D=D, F=F, ...)``: x and dY are their first m
    rows; the gate and up W and B their first f rows; the down W and A their first f columns.  Only the
    slices that are prefixes of a row-major stream are drawn short; the down weight and its A are drawn in
    full and sliced.  Returned like ``make_chain_inputs`` with F = f.
    """
    D = CHAIN["D"] if D is None else D
    F = CHAIN["F"] if F is None else F
    r = CHAIN["r"] if r is None else r
    s = CHAIN["s"] if s is None else s
    w_std = CHAIN["w_std"] if w_std is None else w_std
    if not (0 < f <= F and f % 64 == 0):
        raise ValueError("f must be a positive multiple of 64 not above F")
    x = draw_x(_streams(0), m, D)
    layers = {}
    for name, seed in (("gate", 2), ("up", 3)):
        st = _streams(seed)
        W = draw_w(st, f, D, w_std)                 # first f rows of [F, D]
        A, _ = draw_lora(st, 0, D, r)               # A [r, D] does not depend on F
        B = to_bf16(st[4].standard_normal((f, r), dtype=np.float32) * np.float32(0.01))  # first f rows of [F, r]
        layers[name] = dict(W=W, A=A, B=B, s=s, N=f, K=D, r=r)
    st = _streams(4)
    W = np.ascontiguousarray(draw_w(st, D, F, w_std)[:, :f])
    A, B = draw_lora(st, D, F, r)
    layers["down"] = dict(W=W, A=A[:, :f].contiguous(), B=B, s=s, N=D, K=f, r=r)
    dy = draw_dy(m, D, 1)
    return dict(x=x, dy=dy, layers=layers, M=m, D=D, F=f, r=r, s=s)
