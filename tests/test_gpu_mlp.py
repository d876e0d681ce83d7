"""GPU parity of the SwiGLU kernels and of the gated-MLP block (gate/up -> SwiGLU -> down) against the oracle.

The oracle runs the block as three separate layers with the activations rounded to bf16 between them
(its reading of how the block stores activations); the library fuses gate and up into one stacked layer whose
rows interleave the two by 16, with the SwiGLU in its GEMM epilogue.
"""

import numpy as np
import pytest
import torch

from oracle import linear as L
from oracle import nf4 as O
from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import assert_close, dev, f64, oracle_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 1000, 65537])
def test_swiglu_elementwise(ops, n):
    rng = np.random.default_rng(n)
    g, u, dh = (bf16(rng.standard_normal(n) * 3) for _ in range(3))
    if n:
        g[0] = 40.0  # saturated sigmoid
        g[-1] = -40.0
    h = ops.swiglu_fwd(dev(g), dev(u))
    dg, du = ops.swiglu_bwd(dev(dh), dev(g), dev(u))
    if n == 0:
        return
    assert_close(h, L.swiglu_forward(f64(g), f64(u)), "h")
    rg, ru = L.swiglu_backward(f64(dh), f64(g), f64(u))
    assert_close(dg, rg, "dg")
    assert_close(du, ru, "du")


@pytest.mark.parametrize("M,F", [(1, 8), (37, 264), (300, 1024)])
def test_swiglu_gated(ops, M, F):
    rng = np.random.default_rng(M + F)
    gu = bf16(rng.standard_normal((M, 2 * F)) * 3)
    dh = bf16(rng.standard_normal((M, F)))
    h = ops.swiglu_gated_fwd(dev(gu))
    dgu = ops.swiglu_gated_bwd(dev(dh), dev(gu))
    g, u = f64(gu)[:, :F], f64(gu)[:, F:]
    assert_close(h, L.swiglu_forward(g, u), "h")
    rg, ru = L.swiglu_backward(f64(dh), g, u)
    assert_close(dgu[:, :F], rg, "dg")
    assert_close(dgu[:, F:], ru, "dup")


def build_block(ops, c):
    from qlora_fine_tuning_blockwise_b200.mlp import QLoRAGatedMLP
    Ls = c["layers"]
    return QLoRAGatedMLP(dev(Ls["gate"]["W"]), dev(Ls["up"]["W"]), dev(Ls["down"]["W"]),
                         dev(Ls["gate"]["A"]), dev(Ls["gate"]["B"]), dev(Ls["up"]["A"]), dev(Ls["up"]["B"]),
                         dev(Ls["down"]["A"]), dev(Ls["down"]["B"]), c["s"])


def gate_up_columns(F):
    """Columns of the stacked gate/up output that hold gate feature f and up feature f: the stacked rows are
    interleaved by 16 (16 gate rows, then the 16 up rows of the same features)."""
    f = torch.arange(F, device="cuda")
    gp = (f // 16) * 32 + f % 16
    return gp, gp + 16


def check_grads(grads, rgrads, F):
    """dA, dB of each layer against the oracle; the gate and up dB come as [F / 16, 16, r] views of the stacked
    gradient (feature 16 q + i at [q, i])."""
    for name in ("gate", "up", "down"):
        dA, dB = grads[name]
        if name != "down":
            assert dB.shape[:2] == (F // 16, 16)
            dB = dB.reshape(F, -1)
        assert_close(dA, rgrads[name][0], f"dA {name}")
        assert_close(dB, rgrads[name][1], f"dB {name}")


def oracle_layers(c):
    out = {}
    for name, Ld in c["layers"].items():
        out[name] = (oracle_weight(Ld["W"]), f64(Ld["A"]), f64(Ld["B"]), Ld["s"])
    return out


@pytest.mark.parametrize("M,D,F,r", [(64, 256, 512, 8), (300, 320, 320, 16), (130, 256, 1024, 64)])
def test_gated_mlp_block_small(ops, M, D, F, r):
    c = I.make_chain_inputs(M=M, D=D, F=F, r=r, s=2.0, w_std=0.05)
    block = build_block(ops, c)
    x, dy = dev(c["x"]), dev(c["dy"])
    y, saved = block.forward(x)
    dx, grads = block.backward(dy, x, saved)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    Lo = oracle_layers(c)
    ry, g, u, h = L.mlp_chain_forward(f64(c["x"]), Lo["gate"], Lo["up"], Lo["down"])
    rdx, rgrads = L.mlp_chain_backward(f64(c["dy"]), f64(c["x"]), Lo["gate"], Lo["up"], Lo["down"], (g, u, h))
    gp, up = gate_up_columns(F)
    assert_close(saved[0][:, gp], g, "g")
    assert_close(saved[0][:, up], u, "up")
    assert_close(saved[2], h, "h")
    assert_close(y, ry, "y")
    assert_close(dx, rdx, "dX")
    check_grads(grads, rgrads, F)


def test_gated_mlp_block_full_size_sampled(ops):
    """The 70B-like block (x [8192, 8192], F = 28672, r = 64): y and dX on 64 sampled token rows of the full
    batch; every adapter gradient in full on a 256-token sub-batch run through the same kernels."""
    c = I.make_chain_inputs()
    block = build_block(ops, c)
    Lo = oracle_layers(c)
    x, dy = dev(c["x"]), dev(c["dy"])
    y, saved = block.forward(x)
    dx, _ = block.backward(dy, x, saved)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    rows = np.sort(np.random.default_rng(3).choice(c["M"], size=64, replace=False))
    idx = torch.from_numpy(rows).cuda()
    xs, dys = f64(c["x"])[rows], f64(c["dy"])[rows]
    ry, g, u, h = L.mlp_chain_forward(xs, Lo["gate"], Lo["up"], Lo["down"])
    rdx, _ = L.mlp_chain_backward(dys, xs, Lo["gate"], Lo["up"], Lo["down"], (g, u, h))
    assert_close(y[idx], ry, "y rows")
    assert_close(dx[idx], rdx, "dX rows")
    del y, dx, saved
    # adapter gradients reduce over tokens: check them on a sub-batch of 256 tokens
    Ms = 256
    xs, dys = x[:Ms].contiguous(), dy[:Ms].contiguous()
    ys, saved_s = block.forward(xs)
    _, grads = block.backward(dys, xs, saved_s)
    torch.cuda.synchronize()
    ry, g, u, h = L.mlp_chain_forward(f64(c["x"])[:Ms], Lo["gate"], Lo["up"], Lo["down"])
    _, rgrads = L.mlp_chain_backward(f64(c["dy"])[:Ms], f64(c["x"])[:Ms], Lo["gate"], Lo["up"], Lo["down"], (g, u, h))
    check_grads(grads, rgrads, c["F"])
