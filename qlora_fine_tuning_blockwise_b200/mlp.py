"""Gated MLP block of QLoRA layers: gate and up projections, SwiGLU, down projection, forward and backward.

The gate and up projections read the same input, so they run as ONE QLoRA layer over the stacked weight
[W_gate; W_up] (N = 2F) with rank 2r adapters A = [A_gate; A_up] and block-diagonal B = diag(B_gate, B_up):
its output row is [g | up], and in the backward its dX is dg W_gate + dup W_up + s (dg B_gate) A_gate +
s (dup B_up) A_up -- the sum the block needs -- from a single fused kernel.  The diagonal blocks of its dB
are the gate and up dB; the off-diagonal blocks (gradients of B's structural zeros) are discarded.

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
        W_gu = torch.cat([W_gate, W_up], 0).contiguous()
        A_gu = torch.cat([A_gate, A_up], 0).contiguous()
        B_gu = torch.zeros(2 * F, 2 * r, dtype=torch.bfloat16, device=dev)
        B_gu[:F, :r] = B_gate
        B_gu[F:, r:] = B_up
        self.gate_up = ops.QLoRALinear(W_gu, A_gu, B_gu, s)
        del W_gu
        self.down = ops.QLoRALinear(W_down.contiguous(), A_down, B_down, s)
        self._h = {}
        self._dgu = {}

    def _buf(self, cache, M, shape, dev):
        t = cache.get(M)
        if t is None:
            t = torch.empty(*shape, dtype=torch.bfloat16, device=dev)
            cache[M] = t
        return t

    def forward(self, x: torch.Tensor):
        """y [M, D] bf16 and the activations the backward needs.  Output buffers are reused per M."""
        M = x.shape[0]
        gu, su_gu = self.gate_up.forward(x)
        h = ops.swiglu_gated_fwd(gu, self._buf(self._h, M, (M, self.F), x.device))
        y, su_d = self.down.forward(h)
        return y, (gu, su_gu, h, su_d)

    def backward(self, dy: torch.Tensor, x: torch.Tensor, saved):
        """dX [M, D] bf16 and {"gate"|"up"|"down": (dA fp32, dB fp32)}."""
        gu, su_gu, h, su_d = saved
        M = dy.shape[0]
        dh, dA_d, dB_d = self.down.backward(dy, h, su=su_d)
        dgu = ops.swiglu_gated_bwd(dh, gu, self._buf(self._dgu, M, (M, 2 * self.F), dy.device))
        dx, dA_gu, dB_gu = self.gate_up.backward(dgu, x, su=su_gu)
        F, r = self.F, self.r
        grads = {"gate": (dA_gu[:r], dB_gu[:F, :r]), "up": (dA_gu[r:], dB_gu[F:, r:]), "down": (dA_d, dB_d)}
        return dx, grads

    @staticmethod
    def flops(M: int, D: int, F: int, r: int) -> tuple[int, int]:
        """Algorithmic (fwd, bwd) FLOPs of the block: three QLoRA layers of rank r (SwiGLU not counted)."""
        def fwd(M, N, K):
            return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r

        def bwd(M, N, K):
            return 2 * M * N * K + 2 * M * N * r + 2 * M * r * K + 2 * r * M * K + 2 * N * M * r
        return (2 * fwd(M, F, D) + fwd(M, D, F), 2 * bwd(M, F, D) + bwd(M, D, F))
