"""The NVFP4 forward on the block-scaled FP4 tensor core (qlora_linear_fwd_fp4) against the oracle.

- The weight's scales laid out for the tensor core (nvfp4_scales_to_mma) equal an index-by-index re-layout of the
  row-major scales done here on the CPU: the atoms of 128 rows x 4 groups, byte 16 (row % 32) + 4 (row % 128 / 32)
  + group, padded rows and steps zero.
- The activations quantized inside the call (codes, scales, tensor scale) equal the oracle's NVFP4 quantization of
  the same bf16 values, bit for bit.
- y equals the oracle's FP4 form of the layer (reading R24: q(x) q(W)^T + s (x A^T) B^T, fp64) within the GEMM
  tolerance, on ragged shapes, without and with the LoRA term, and on operands whose rows and 16-groups span many
  binades, so that a scale applied to the wrong row or group cannot go unnoticed.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4 as F
from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import assert_close, dev, f64, lora_or_none

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def mma_layout(scales_rowmajor: np.ndarray, rows: int, K: int) -> np.ndarray:
    """The MMA scale layout built on the CPU, one byte at a time."""
    groups = K // 16
    steps = (K + 255) // 256 * 4
    rb = (rows + 127) // 128
    out = np.zeros(rb * steps * 512, dtype=np.uint8)
    sc = scales_rowmajor.reshape(rows, groups)
    for r in range(rows):
        for g in range(groups):
            rr = r % 128
            off = (r // 128) * steps * 512 + (g // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + (g % 4)
            out[off] = sc[r, g]
    return out


def from_mma_layout(sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Row-major scales [rows, K/16] read back from the MMA layout (the inverse of mma_layout)."""
    groups = K // 16
    steps = (K + 255) // 256 * 4
    r = np.arange(rows)[:, None]
    g = np.arange(groups)[None, :]
    rr = r % 128
    off = (r // 128) * steps * 512 + (g // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + (g % 4)
    return sf[off]


@pytest.mark.parametrize("rows,K", [(1, 64), (128, 256), (300, 640), (257, 1088)])
def test_weight_scales_mma_layout(ops, rows, K):
    rng = np.random.default_rng(rows + K)
    W = (rng.standard_normal((rows, K)) * np.exp2(rng.integers(-6, 6, size=(rows, 1)))).astype(np.float32)
    codes, scales, S = ops.nvfp4_quantize(dev(W))
    sf = ops.nvfp4_scales_to_mma(scales, rows, K)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    expect = mma_layout(scales.cpu().numpy(), rows, K)
    assert sf.numel() == expect.size
    assert np.array_equal(sf.cpu().numpy(), expect)


CASES = [(64, 256, 256, 8), (300, 264, 640, 72), (16, 1024, 2048, 16), (128, 512, 1024, 0), (200, 136, 1088, 64),
         (2048, 4096, 4096, 16)]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_fp4_forward_against_oracle(ops, M, N, K, r):
    d = I.make_random_linear(M, N, K, r, s=2.0, seed=M + N + K + r)
    layer = ops.FP4Linear(dev(d["W"]), *lora_or_none(d), 2.0)
    y, su = layer.forward(dev(d["x"]), want_su=True)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    x32 = d["x"].float().numpy()
    # the activations as the call quantized them, bit for bit
    codes, sf, S = layer.quantized_activations(M)
    rc, rs, rS = F.nvfp4_quantize(x32)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(from_mma_layout(sf.cpu().numpy(), M, K).reshape(-1), rs)
    assert S.item() == float(rS)
    A, B = (None, None) if r == 0 else (f64(d["A"]), f64(d["B"]))
    ref = F.fp4_linear_forward(x32, d["W"], A, B, 2.0)
    assert_close(y, ref, f"y fp4 {M}x{N}x{K} r{r}")


def test_fp4_forward_scales_reach_the_right_rows_and_groups(ops):
    """Rows of W and of x and their 16-element groups at magnitudes 2^-8 .. 2^8 apart: each output mixes
    contributions whose sizes differ by orders of magnitude, so a scale taken from another row or group would
    move y far outside the tolerance."""
    M, N, K, r = 192, 320, 512, 0
    rng = np.random.default_rng(7)
    W = rng.standard_normal((N, K)).astype(np.float32)
    W *= np.exp2(rng.integers(-8, 9, size=(N, 1))).astype(np.float32)
    W *= np.exp2(rng.integers(-4, 5, size=(1, K // 16))).repeat(16, axis=1).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x *= np.exp2(rng.integers(-8, 9, size=(M, 1))).astype(np.float32)
    x *= np.exp2(rng.integers(-4, 5, size=(M, K // 16))).repeat(16, axis=1).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    layer = ops.FP4Linear(dev(W), None, None, 1.0)
    y, _ = layer.forward(dev(xb))
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    ref = F.fp4_linear_forward(xb.float().numpy(), W, None, None, 1.0)
    # row by row, since the rows' magnitudes differ by up to 2^16
    yg = f64(y)
    for m in range(M):
        assert_close(yg[m], ref[m], f"row {m}")


def test_fp4_forward_rejects_bad_arguments(ops):
    import ctypes
    L = ops.lib()
    p = ctypes.c_void_p(0x10000)
    assert L.qlora_linear_fwd_fp4(64, 256, 100, 8, p, p, p, p, p, p, 2.0, p, None, p, 1 << 30, None) == ops.QL_ERR_INVALID_ARG
    assert L.qlora_linear_fwd_fp4(64, 256, 256, 8, p, p, p, p, p, p, 2.0, p, None, p, 16, None) == ops.QL_ERR_INVALID_ARG
    assert L.nvfp4_scales_to_mma(p, 4, 96, p, None) == ops.QL_ERR_INVALID_ARG
