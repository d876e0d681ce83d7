"""The gated MLP's fused SwiGLU epilogues against the unfused path, bit for bit: the gate/up GEMM that writes h in
its epilogue against the plain GEMM followed by the elementwise SwiGLU kernel, and the down projection's dX GEMM that
writes dgu in its epilogue against the plain dX GEMM followed by the elementwise SwiGLU backward."""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def positions(F):
    f = torch.arange(F, device="cuda")
    gp = (f // 16) * 32 + f % 16
    return gp, gp + 16


@pytest.mark.parametrize("M,F,D,r", [(256, 512, 256, 8), (300, 320, 320, 16), (16, 1024, 512, 16), (2048, 2048, 1024, 64)])
def test_fused_forward_and_backward_equal_the_unfused_path(ops, M, F, D, r):
    from qlora_fine_tuning_blockwise_b200.mlp import QLoRAGatedMLP
    c = I.make_chain_inputs(M=M, D=D, F=F, r=r)
    Ls = c["layers"]
    block = QLoRAGatedMLP(dev(Ls["gate"]["W"]), dev(Ls["up"]["W"]), dev(Ls["down"]["W"]), dev(Ls["gate"]["A"]),
                          dev(Ls["gate"]["B"]), dev(Ls["up"]["A"]), dev(Ls["up"]["B"]), dev(Ls["down"]["A"]),
                          dev(Ls["down"]["B"]), c["s"])
    x, dy = dev(c["x"]), dev(c["dy"])
    y, (gu, su_gu, h, su_d) = block.forward(x)
    gp, up = positions(F)
    # unfused forward: the plain layer call, then the elementwise SwiGLU of the de-interleaved halves
    gu2, _ = block.gate_up.forward(x)
    assert torch.equal(gu2.view(torch.int16), gu.view(torch.int16))
    h2 = ops.swiglu_fwd(gu2[:, gp].contiguous(), gu2[:, up].contiguous())
    assert torch.equal(h2.view(torch.int16), h.view(torch.int16))
    # unfused backward of the down projection: dh, then the elementwise SwiGLU backward
    dx_fused, _ = block.backward(dy, x, (gu, su_gu, h, su_d))
    dh, _, _ = block.down.backward(dy, h, su=su_d)
    dg, du = ops.swiglu_bwd(dh, gu[:, gp].contiguous(), gu[:, up].contiguous())
    dgu = block._dgu[M]
    assert torch.equal(dgu[:, gp].view(torch.int16), dg.view(torch.int16))
    assert torch.equal(dgu[:, up].view(torch.int16), du.view(torch.int16))
    assert ops.device_error() == ops.QL_OK
