"""GPU parity of the weight-format conversions against the oracle: double-quantized NF4 block constants and NVFP4.

Both are bit-exact: every step is one IEEE operation in a fixed order on both sides (``oracle.double_quant``,
``oracle.nvfp4``).  The cases are:
- ragged group counts, constant and zero inputs;
- the constants of a real NF4 weight;
- the 28672 x 8192 decode-layer weight: all of its 3.67M block constants, and a sample of its NVFP4 blocks
  that holds the tensor's largest weight;
- bf16 outputs;
- the device error word on non-finite input.

This file is collected last, so that a failure here stops a run only after every other test has run.
"""

import numpy as np
import pytest
import torch

from oracle import double_quant as D
from oracle import nf4 as O
from oracle import nvfp4 as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def bits(t):
    return t.cpu().numpy().view(np.uint32) if t.dtype == torch.float32 else t.cpu().numpy()


# ------------------------------------------------------------------ double quantization


def check_dq(ops, c):
    code8, c1, mu = ops.nf4_double_quantize(torch.from_numpy(c).cuda())
    back = ops.nf4_double_dequantize(code8, c1, mu)
    q, c1o, muo = D.dq_quantize(c)
    assert ops.formats_device_error() == ops.QL_OK
    assert bits(mu)[0] == np.float32(muo).view(np.uint32)
    assert np.array_equal(code8.cpu().numpy(), q)
    assert np.array_equal(bits(c1), c1o.view(np.uint32))
    assert np.array_equal(bits(back), D.dq_dequantize(q, c1o, muo).view(np.uint32))


@pytest.mark.parametrize("nb,seed", [(1, 0), (255, 1), (256, 2), (257, 3), (256 * 37 + 5, 4)])
def test_double_quantization_random(ops, nb, seed):
    check_dq(ops, np.random.default_rng(seed).uniform(0.005, 0.09, nb).astype(np.float32))


def test_double_quantization_special(ops):
    k = np.arange(15)
    for c in (np.full(700, 0.0371, np.float32), np.zeros(300, np.float32),
              np.concatenate([1 + 2.0 ** -k / 2, 1 - 2.0 ** -k / 2]).astype(np.float32)):
        check_dq(ops, c)


def test_double_quantization_of_a_decode_layer(ops):
    """All 3.67M block constants of the 28672 x 8192 weight, as nf4_quantize writes them on the device."""
    W = (np.random.default_rng(2).standard_normal((28672, 8192)) * 0.015).astype(np.float32)
    _, absmax = ops.nf4_quantize(torch.from_numpy(W).cuda())
    check_dq(ops, absmax.cpu().numpy())


# ------------------------------------------------------------------ NVFP4


def check_fp4(ops, W):
    w = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    codes, scales, S = ops.nvfp4_quantize(w)
    co, so, So = F.nvfp4_quantize(W)
    assert ops.formats_device_error() == ops.QL_OK
    assert bits(S)[0] == So.view(np.uint32)
    assert np.array_equal(scales.cpu().numpy(), so)
    assert np.array_equal(codes.cpu().numpy(), co)
    want = F.nvfp4_dequantize(co, so, So, W.size)
    back = ops.nvfp4_dequantize(codes, scales, S, W.size)
    assert np.array_equal(bits(back), want.view(np.uint32))
    back16 = ops.nvfp4_dequantize(codes, scales, S, W.size, dtype=torch.bfloat16)
    want16 = O.f32_to_bf16_bits(want)
    assert np.array_equal(back16.view(torch.int16).cpu().numpy().view(np.uint16), want16)


@pytest.mark.parametrize("rows,cols,std,seed", [(1, 16, 0.015, 0), (3, 48, 1.0, 1), (64, 512, 0.015, 2),
                                                (17, 1024, 0.003, 3), (1000, 4096, 0.015, 4)])
def test_nvfp4_random(ops, rows, cols, std, seed):
    check_fp4(ops, (np.random.default_rng(seed).standard_normal((rows, cols)) * std).astype(np.float32))


def test_nvfp4_zero_blocks_and_signs(ops):
    W = (np.random.default_rng(7).standard_normal(40 * 16) * 0.02).astype(np.float32)
    W[32:48] = 0.0
    W[50] = -0.0
    W[60:64] *= 1e-6
    W[5] = 0.5
    check_fp4(ops, W)
    check_fp4(ops, np.zeros(64, np.float32))


def test_nvfp4_decode_layer_sampled(ops):
    """The 28672 x 8192 weight quantized whole on the device; 64 sampled rows plus the row of the tensor's largest
    weight are checked against the oracle, which sees the same largest magnitude and hence the same S."""
    W = (np.random.default_rng(8).standard_normal((28672, 8192)) * 0.015).astype(np.float32)
    codes, scales, S = ops.nvfp4_quantize(torch.from_numpy(W).cuda())
    top = int(np.argmax(np.abs(W)) // W.shape[1])
    rows = np.unique(np.concatenate([np.random.default_rng(9).integers(0, W.shape[0], 64), [top]]))
    co, so, So = F.nvfp4_quantize(W[rows])
    assert bits(S)[0] == So.view(np.uint32)
    c = codes.view(W.shape[0], W.shape[1] // 2).cpu().numpy()[rows].reshape(-1)
    s = scales.view(W.shape[0], W.shape[1] // 16).cpu().numpy()[rows].reshape(-1)
    assert np.array_equal(c, co) and np.array_equal(s, so)


def test_nonfinite_input_is_reported(ops):
    W = np.zeros(64, np.float32)
    W[7] = np.nan
    ops.nvfp4_quantize(torch.from_numpy(W).cuda())
    assert ops.formats_device_error() == ops.QL_ERR_INVALID_ARG
    assert ops.formats_device_error() == ops.QL_OK  # read-and-clear


def test_launches_are_counted(ops):
    n0 = ops.formats_launch_count()
    ops.nvfp4_quantize(torch.ones(32, device="cuda"))
    assert ops.formats_launch_count() - n0 == 3
