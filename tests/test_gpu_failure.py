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
