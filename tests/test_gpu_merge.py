"""GPU parity of the LoRA merge (W' = deq(W) + s B A) and its NF4 requantization against the oracle: bit-exact,
since both sides take every fp32 step in the same order (see ``oracle.merge``)."""

import numpy as np
import pytest
import torch

from oracle import merge as M
from oracle import nf4 as O
from tests.gpu_common import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def layer(N, K, r, seed, w_std=0.02):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * w_std).astype(np.float32)
    codes, absmax = O.nf4_quantize(W)
    A = O.round_bf16(rng.standard_normal((r, K)).astype(np.float32) / np.sqrt(K))
    B = O.round_bf16(rng.standard_normal((N, r)).astype(np.float32) * 0.05)
    return codes, absmax, A, B


def to_dev(codes, absmax, A, B):
    c = torch.from_numpy(codes).cuda()
    a = torch.from_numpy(absmax).cuda()
    At = torch.from_numpy(A).to(torch.bfloat16).cuda() if A.shape[0] else None
    Bt = torch.from_numpy(B).to(torch.bfloat16).cuda() if A.shape[0] else None
    return c, a, At, Bt


CASES = [
    # N, K, r, s
    (1, 64, 0, 2.0),        # no adapter: W' = deq(W)
    (3, 192, 1, 2.0),
    (37, 256, 16, 0.5),
    (5, 128, 17, -1.5),     # rank not a multiple of 8, negative scaling
    (130, 512, 64, 2.0),
    (64, 1024, 256, 1.0),   # largest rank
]


@pytest.mark.parametrize("N,K,r,s", CASES)
def test_merge_bit_exact(ops, N, K, r, s):
    codes, absmax, A, B = layer(N, K, r, seed=N + K + r)
    c, a, At, Bt = to_dev(codes, absmax, A, B)
    w32 = ops.merge_lora(c, a, At, Bt, s, N, K, dtype=torch.float32)
    w16 = ops.merge_lora(c, a, At, Bt, s, N, K, dtype=torch.bfloat16)
    c2, a2 = ops.merge_lora_nf4(c, a, At, Bt, s, N, K)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    ref = M.merge_lora(codes, absmax, A, B, s, N, K)
    assert np.array_equal(w32.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(w16.view(torch.int16).cpu().numpy().view(np.uint16), M.merge_lora_bf16_bits(codes, absmax, A, B, s, N, K))
    rc, ra = M.merge_lora_nf4(codes, absmax, A, B, s, N, K)
    assert np.array_equal(c2.cpu().numpy(), rc)
    assert np.array_equal(a2.cpu().numpy().view(np.uint32), ra.view(np.uint32))


def test_merge_in_place_equals_out_of_place(ops):
    N, K, r, s = 96, 640, 32, 2.0
    codes, absmax, A, B = layer(N, K, r, seed=3)
    c, a, At, Bt = to_dev(codes, absmax, A, B)
    c2, a2 = ops.merge_lora_nf4(c, a, At, Bt, s, N, K)
    ops.merge_lora_nf4(c, a, At, Bt, s, N, K, codes_out=c, absmax_out=a)  # in place
    torch.cuda.synchronize()
    assert torch.equal(c, c2) and torch.equal(a, a2)


def test_zero_adapter_gives_back_the_base(ops):
    N, K, r = 40, 384, 8
    codes, absmax, A, B = layer(N, K, r, seed=4)
    c, a, At, _ = to_dev(codes, absmax, A, B)
    B0 = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    c2, a2 = ops.merge_lora_nf4(c, a, At, B0, 2.0, N, K)
    w = ops.merge_lora(c, a, At, B0, 2.0, N, K)
    torch.cuda.synchronize()
    assert torch.equal(c2, c) and torch.equal(a2, a)
    assert torch.equal(w, ops.nf4_dequantize(c, a, N * K).view(N, K))


def test_merge_attention_layer_full(ops):
    """A 4096 x 4096 layer with rank 16, every element compared."""
    N, K, r, s = 4096, 4096, 16, 2.0
    codes, absmax, A, B = layer(N, K, r, seed=5)
    c, a, At, Bt = to_dev(codes, absmax, A, B)
    c2, a2 = ops.merge_lora_nf4(c, a, At, Bt, s, N, K)
    torch.cuda.synchronize()
    rc, ra = M.merge_lora_nf4(codes, absmax, A, B, s, N, K)
    assert np.array_equal(c2.cpu().numpy(), rc)
    assert np.array_equal(a2.cpu().numpy().view(np.uint32), ra.view(np.uint32))
