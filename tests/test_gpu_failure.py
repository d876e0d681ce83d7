"""Failure detection on the GPU without a fault: every wait in the kernels is bounded.

ql_selftest_wait_timeout launches one kernel whose thread waits on an mbarrier that nothing arrives on,
through the same bounded-wait routine the GEMM kernels use, with a ~1 ms limit.  The wait must give up,
the kernel must return normally, the host must read QL_ERR_TIMEOUT from the device error word, and the
context must stay usable.  Nothing here traps, faults or hangs the GPU.
"""

import numpy as np
import pytest
import torch

from oracle import nf4 as O
from tests.gpu_common import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def test_bounded_wait_reports_timeout_and_context_survives(ops):
    assert ops.device_error() == ops.QL_OK
    ops.selftest_wait_timeout(2_000_000)
    assert ops.device_error() == ops.QL_ERR_TIMEOUT
    assert ops.device_error() == ops.QL_OK  # reading clears the word
    w = np.random.default_rng(0).standard_normal(64 * 33).astype(np.float32)
    codes, absmax = ops.nf4_quantize(dev(w))
    c_ref, a_ref = O.nf4_quantize(w)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert ops.device_error() == ops.QL_OK


def test_nonfinite_weight_is_reported(ops):
    w = np.zeros(128, np.float32)
    w[70] = np.inf
    ops.nf4_quantize(dev(w))
    assert ops.device_error() == ops.QL_ERR_INVALID_ARG
    assert ops.device_error() == ops.QL_OK


def test_selftest_rejects_bad_limit(ops):
    with pytest.raises(ops.QLoRAError):
        ops.selftest_wait_timeout(0)


@pytest.mark.parametrize("role,r,which", [(1, 16, "fwd"), (2, 16, "fwd"), (3, 0, "fwd"),
                                          (1, 16, "dx"), (2, 16, "dx"), (3, 0, "dx")])
def test_fused_gemm_abort_path(ops, role, r, which):
    """One warp role of the fused GEMM (1 the MMA issuer, 2 the activation producer, 3 the codes producer) leaves
    before doing anything, with every wait bounded at ~10 ms: the other roles' waits expire, the kernel drains
    what it issued, frees tensor memory and returns; the host reads QL_ERR_TIMEOUT, and the next call of the
    same layer gives the same result as before, bit for bit."""
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    from tests.gpu_common import lora_or_none
    M, N, K = 300, 264, 640
    d = I.make_random_linear(M, N, K, r, s=2.0, seed=40 + role)
    layer = ops.QLoRALinear(dev(d["W"]), *lora_or_none(d), 2.0)
    x, dy = dev(d["x"]), dev(d["dy"])
    y, su = layer.forward(x)
    y_ref, su_ref = y.clone(), (su.clone() if su is not None else None)
    dx, _, _ = layer.backward(dy, x, su=su_ref)
    dx_ref = dx.clone()
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    ops.selftest_arm_gemm_stall(role, 20_000_000)
    if which == "fwd":
        layer.forward(x)
    else:
        layer.backward(dy, x, su=su_ref)
    assert ops.device_error() == ops.QL_ERR_TIMEOUT
    assert ops.device_error() == ops.QL_OK
    y2, _ = layer.forward(x)
    dx2, _, _ = layer.backward(dy, x, su=su_ref)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    assert torch.equal(y2, y_ref) and torch.equal(dx2, dx_ref)


def test_gemm_stall_hook_rejects_bad_arguments(ops):
    with pytest.raises(ops.QLoRAError):
        ops.selftest_arm_gemm_stall(0, 20_000_000)
    with pytest.raises(ops.QLoRAError):
        ops.selftest_arm_gemm_stall(1, 10)
