"""The fused GEMMs on double-quantized NF4 and NVFP4 base weights against the oracle: the weight is dequantized by
the oracle's own format rules (double-quantized block constants, or E2M1 codes with E4M3 group scales) and the layer
computed in fp64; the GPU reads the compressed format inside its GEMMs."""
import numpy as np
import pytest
import torch

from oracle import double_quant as D
from oracle import linear as L
from oracle import nf4 as O
from oracle import nvfp4 as F
from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import assert_close, dev, f64, lora_or_none

pytestmark = pytest.mark.gpu
CASES = [(64, 256, 256, 8), (300, 320, 640, 16), (16, 1024, 2048, 16), (2048, 4096, 4096, 16)]


@pytest.mark.parametrize("fmt", ["nf4_dq", "nvfp4"])
@pytest.mark.parametrize("M,N,K,r", CASES)
def test_forward_backward_against_oracle(fmt, M, N, K, r):
    from qlora_fine_tuning_blockwise_b200 import ops
    d = I.make_linear_inputs(I.LinearWorkload("t", M, K, N, r, 2.0, 0.02))
    W = d["W"]
    w = getattr(ops.Weight, fmt)(dev(W))
    if fmt == "nf4_dq":
        codes, absmax = O.nf4_quantize(W)
        q, c1, mu = D.dq_quantize(absmax)
        Wd = O.nf4_dequantize(codes, D.dq_dequantize(q, c1, mu), N * K).reshape(N, K).astype(np.float64)
    else:
        c, sb, S = F.nvfp4_quantize(W)
        Wd = F.nvfp4_dequantize(c, sb, S, N * K).reshape(N, K).astype(np.float64)
    A, B = lora_or_none(d)
    x, dy = dev(d["x"]), dev(d["dy"])
    y, su = ops.linear_fwd_w(x, w, A, B, d["s"])
    dx, dA, dB = ops.linear_bwd_w(dy, x, w, A, B, d["s"], su=su)
    torch.cuda.synchronize()
    xs, dys, As, Bs = f64(d["x"]), f64(d["dy"]), f64(d["A"]), f64(d["B"])
    assert_close(y, L.qlora_forward(xs, Wd, As, Bs, d["s"]), f"{fmt} y")
    rdx, rdA, rdB = L.qlora_backward(dys, xs, Wd, As, Bs, d["s"])
    assert_close(dx, rdx, f"{fmt} dX")
    if r:
        assert_close(dA, rdA, f"{fmt} dA")
        assert_close(dB, rdB, f"{fmt} dB")
