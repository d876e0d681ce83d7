"""Gated MLP block of QLoRA layers: gate and up projections, SwiGLU, down projection, forward and backward.

The gate and up projections read the same input, so they run as ONE QLoRA layer over the stacked weight of
W_gate and W_up (N = 2F) with rank 2r adapters A = [A_gate; A_up] and block-diagonal B: its dX is
dg W_gate + dup W_up + s (dg B_gate) A_gate + s (dup B_up) A_up -- the sum the block needs -- from one fused
kernel.  The stacked rows are INTERLEAVED by 16 (16 gate rows, then the 16 up rows of the same features), so
that the GEMM epilogue that writes gu also holds g and up of a feature in two lanes of one warp and writes
h = silu(g) * up itself; the down projection's dX epilogue likewise turns dh into dgu.  Neither h's input gu
nor dh makes an extra round trip through HBM.  The gate and up dB are strided views of the stacked dB (its
off-diagonal blocks, the gradients of B's structural zeros, are ignored).

Per "Inside Unsloth: How the Fastest LLM Fine-Tuning Library Works" (thriftbooks.com), section "What You'll
Learn", item "Triton Kernel Internals" (fused SwiGLU forward/backward) and "unsloth" (pyshine.com), the
kernels-directory paragraph (swiglu.py fuses the gated MLP activation; fast_lora.py the LoRA matmuls).

Activations g, up, h and the gradients dh, dg, dup cross the kernels in bf16, as a fine-tuning framework
stores them.  Everything on the step runs in libqlora's kernels; torch only allocates and, once at
construction, lays the parameters out (stacking, block-diagonal B).
"""

from __future__ import annotations

import torch

from . import ops


class QLoRAGatedMLP:
    def __init__(self, W_gate, W_up, W_down, A_gate, B_gate, A_up, B_up, A_down, B_down, s: float):
        F, D = W_gate.shape
        r = A_gate.shape[0]
        dev = W_gate.device
        self.D, self.F, self.r, self.s = D, F, r, float(s)
        assert F % 16 == 0, "the interleaved gate/up layout needs F % 16 == 0"
        # row 32q + i: gate feature 16q + i; row 32q + 16 + i: up feature 16q + i (i < 16)
        W_gu = torch.stack([W_gate.reshape(F // 16, 16, D), W_up.reshape(F // 16, 16, D)], 1).reshape(2 * F, D)
        A_gu = torch.cat([A_gate, A_up], 0).contiguous()
        B_gu = torch.zeros(F // 16, 2, 16, 2 * r, dtype=torch.bfloat16, device=dev)
        B_gu[:, 0, :, :r] = B_gate.reshape(F // 16, 16, r)
        B_gu[:, 1, :, r:] = B_up.reshape(F // 16, 16, r)
        self.gate_up = ops.QLoRALinear(W_gu.contiguous(), A_gu, B_gu.reshape(2 * F, 2 * r), s)
        del W_gu
        self.down = ops.QLoRALinear(W_down.contiguous(), A_down, B_down, s)
        self._h = {}
        self._dgu = {}
        # measurement hook: when set, called with "gate_up_fwd", "down_fwd", "down_dx" or "gate_up_dx" just
        # before the call that launches that fused GEMM (the benchmark retargets its profiling events there)
        self.on_kernel = None

    def _mark(self, tag: str) -> None:
        if self.on_kernel is not None:
            self.on_kernel(tag)

    def _buf(self, cache, M, shape, dev):
        t = cache.get(M)
        if t is None:
            t = torch.empty(*shape, dtype=torch.bfloat16, device=dev)
            cache[M] = t
        return t

    def forward(self, x: torch.Tensor):
        """y [M, D] bf16 and the activations the backward needs.  Output buffers are reused per M."""
        M = x.shape[0]
        self._mark("gate_up_fwd")
        gu, h, su_gu = ops.gate_up_fwd_swiglu(x, self.gate_up, self._buf(self._h, M, (M, self.F), x.device))
        self._mark("down_fwd")
        y, su_d = self.down.forward(h)
        return y, (gu, su_gu, h, su_d)

    def backward(self, dy: torch.Tensor, x: torch.Tensor, saved):
        """dX [M, D] bf16 and {"gate"|"up"|"down": (dA fp32, dB fp32)}; the gate and up dB are [F/16, 16, r] views."""
        gu, su_gu, h, su_d = saved
        M = dy.shape[0]
        self._mark("down_dx")
        dgu, dA_d, dB_d = ops.down_bwd_dswiglu(dy, h, self.down, su_d, gu,
                                               self._buf(self._dgu, M, (M, 2 * self.F), dy.device))
        self._mark("gate_up_dx")
        dx, dA_gu, dB_gu = self.gate_up.backward(dgu, x, su=su_gu)
        F, r = self.F, self.r
        # the interleaved rows of the stacked dB as strided views (no copy): [F / 16, 16, r] each, feature
        # 16 q + i at [q, i]; reshape(F, r) gives the plain layout
        dB4 = dB_gu.view(F // 16, 2, 16, 2 * r)
        grads = {"gate": (dA_gu[:r], dB4[:, 0, :, :r]), "up": (dA_gu[r:], dB4[:, 1, :, r:]), "down": (dA_d, dB_d)}
        return dx, grads

    @staticmethod
    def flops(M: int, D: int, F: int, r: int) -> tuple[int, int]:
        """Algorithmic (fwd, bwd) FLOPs of the block: three QLoRA layers of rank r (SwiGLU not counted)."""
        def fwd(M, N, K):
            return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r

        def bwd(M, N, K):
            return 2 * M * N * K + 2 * M * N * r + 2 * M * r * K + 2 * r * M * K + 2 * N * M * r
        return (2 * fwd(M, F, D) + fwd(M, D, F), 2 * bwd(M, F, D) + bwd(M, D, F))
