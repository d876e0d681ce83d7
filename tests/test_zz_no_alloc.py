"""The scratch-free forward (qlora_linear_fwd_noalloc) against the regular forward, through the C ABI.

qlora_linear_fwd_noalloc exists for callers that cannot allocate device memory -- for example code running
under global-mode stream capture, where cudaMalloc is an error, or a plug-in whose host program forbids
device allocation after start-up.  It must give the regular forward's result, also when it is called
twice in a row (its built-in scratch keeps the previous call's contents), and must refuse sizes whose
scratch exceeds its fixed 8 MiB.  This file is collected last so that a failure here stops a run only after
every other test has run.
"""

import ctypes

import pytest
import torch

from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import assert_close, dev, lora_or_none

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


# a decode-sized layer (split contraction for s*x*A^T, so the scratch holds fp32 partial sums), the tiny
# workload, and a ragged multi-tile shape
CASES = [(16, 2048, 8192, 16), (64, 256, 256, 8), (300, 264, 640, 72)]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_noalloc_forward_matches_regular_forward_twice(ops, M, N, K, r):
    assert ops.workspace_bytes(M, N, K, r, ops.QL_PASS_FWD) <= 8 << 20
    results = []
    for seed in (21, 22):  # two calls in a row with different inputs: no stale scratch may leak through
        d = I.make_random_linear(M, N, K, r, s=2.0, seed=seed + M)
        codes, absmax = ops.nf4_quantize(dev(d["W"]))
        x = dev(d["x"])
        A, B = lora_or_none(d)
        y_ref, su_ref = ops.qlora_linear_fwd(x, codes, absmax, A, B, 2.0, N, K)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        su = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda") if r else None
        ops.qlora_linear_fwd_noalloc(x, codes, absmax, A, B, 2.0, N, K, y, su)
        torch.cuda.synchronize()
        assert ops.device_error() == ops.QL_OK
        assert_close(y, y_ref, "y (scratch-free vs regular)")
        assert torch.equal(y, y_ref)
        if r:
            assert_close(su, su_ref, "s*x*A^T (scratch-free vs regular)")
            assert torch.equal(su, su_ref)
        results.append(y)
    assert not torch.equal(results[0], results[1])


def test_noalloc_rejects_sizes_beyond_its_scratch(ops):
    M, N, K, r = 256, 8192, 16384, 8
    assert ops.workspace_bytes(M, N, K, r, ops.QL_PASS_FWD) > 8 << 20
    p = ctypes.c_void_p(0x10000)
    st = ops.lib().qlora_linear_fwd_noalloc(M, N, K, r, p, p, p, p, p, 2.0, p, None, None)
    assert st == ops.QL_ERR_INVALID_ARG
