"""GPU parity of nf4_quantize / nf4_dequantize against the oracle: bit-exact, through the C ABI."""

import numpy as np
import pytest
import torch

from oracle import nf4 as O
from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def check_roundtrip(ops, W: np.ndarray):
    w = dev(np.ascontiguousarray(W, dtype=np.float32).reshape(-1))
    codes, absmax = ops.nf4_quantize(w)
    c_ref, a_ref = O.nf4_quantize(W)
    assert np.array_equal(codes.cpu().numpy(), c_ref), "codes differ"
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32)), "absmax differs"
    n = W.size
    d32 = ops.nf4_dequantize(codes, absmax, n, dtype=torch.float32)
    assert np.array_equal(d32.cpu().numpy().view(np.uint32), O.nf4_dequantize(c_ref, a_ref, n).view(np.uint32))
    d16 = ops.nf4_dequantize(codes, absmax, n, dtype=torch.bfloat16)
    assert np.array_equal(d16.view(torch.int16).cpu().numpy().view(np.uint16),
                          O.nf4_dequantize_bf16_bits(c_ref, a_ref, n))
    assert ops.device_error() == ops.QL_OK


def test_codebook_matches_oracle(ops):
    assert np.array_equal(ops.codebook().view(np.uint32), O.nf4_codebook().view(np.uint32))


@pytest.mark.parametrize("name", ["tiny_64x256x256_r8", "attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64"])
def test_quantize_workload_weights(ops, name):
    w = I.WORKLOADS[name]
    W = I.draw_w(I._streams(0), w.N, w.K, w.w_std)
    check_roundtrip(ops, W)


def test_quantize_decode_weight_sampled_blocks(ops):
    """The 28672 x 8192 weight at full size; blocks are independent, so a sample is checked bit for bit."""
    w = I.WORKLOADS["decode_16x8192x28672_r16"]
    W = I.draw_w(I._streams(0), w.N, w.K, w.w_std)
    codes, absmax = ops.nf4_quantize(dev(W.reshape(-1)))
    rng = np.random.default_rng(0)
    blocks = rng.choice(W.size // 64, size=20000, replace=False)
    blocks.sort()
    flat = W.reshape(-1, 64)[blocks]
    c_ref, a_ref = O.nf4_quantize(flat)
    cg = codes.view(-1, 32)[torch.from_numpy(blocks).cuda()].cpu().numpy().reshape(-1)
    ag = absmax[torch.from_numpy(blocks).cuda()].cpu().numpy()
    assert np.array_equal(cg, c_ref) and np.array_equal(ag.view(np.uint32), a_ref.view(np.uint32))


@pytest.mark.parametrize("nblocks", [1, 3, 97, 1001])
def test_quantize_ragged_block_counts(ops, nblocks):
    W = I.draw_w(I._streams(nblocks), 1, 64 * nblocks, 0.02)
    check_roundtrip(ops, W)


def test_quantize_edge_values(ops):
    """Zero blocks, exact level multiples, midpoints and their fp32 neighbours, both signs, tiny and huge scales."""
    c = O.nf4_codebook()
    mids = (c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2
    vals = []
    for m in mids:
        f = np.float32(m)
        vals += [np.nextafter(f, np.float32(-2)), f, np.nextafter(f, np.float32(2))]
    vals += list(c)
    vals = np.array(vals, dtype=np.float32)
    blocks = []
    for scale in (np.float32(1.0), np.float32(0.5), np.float32(3.0e-3), np.float32(7.5e3), np.float32(1e-30)):
        v = vals * scale
        for start in range(0, v.size, 63):
            chunk = v[start:start + 63]
            blk = np.zeros(64, np.float32)
            blk[0] = scale  # the block maximum -> the normalised values are exactly vals
            blk[1:1 + chunk.size] = chunk
            blocks.append(blk)
    blocks.append(np.zeros(64, np.float32))                 # all-zero block
    blocks.append(-np.abs(blocks[0]))                       # maximum magnitude on a negative element
    W = np.stack(blocks).reshape(1, -1)
    check_roundtrip(ops, W)


def test_quantize_every_fp32_in_unit_interval(ops):
    """Every fp32 bit pattern in [0, 1] and its negative, as the normalised values of blocks whose absmax is 1
    (one element 1.0, then 63 values), in chunks; the expected codes come from the oracle's rule on the same
    values."""
    top = 0x3F800000 + 1          # patterns 0 .. bits(1.0)
    chunk = 63 * (1 << 19)        # whole blocks of 63 values
    one = int(O.nf4_code_of(np.array([1.0], np.float32))[0])
    for p0 in range(0, top, chunk):
        p1 = min(p0 + chunk, top)
        n = p1 - p0
        nb = -(-n // 63)
        host = np.arange(p0, p1, dtype=np.uint32).view(np.float32)
        pats = torch.arange(p0, p1, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32)
        for sign in (1.0, -1.0):
            v = torch.zeros(nb * 63, dtype=torch.float32, device="cuda")
            v[:n] = pats * sign
            W = torch.cat([torch.ones(nb, 1, dtype=torch.float32, device="cuda"), v.view(nb, 63)], dim=1)
            codes, absmax = ops.nf4_quantize(W.reshape(-1).contiguous())
            vh = np.zeros(nb * 63, np.float32)
            vh[:n] = host * np.float32(sign)
            e = O.nf4_code_of(vh).reshape(nb, 63).astype(np.uint8)
            full = np.concatenate([np.full((nb, 1), one, np.uint8), e], axis=1)
            packed = ((full[:, 0::2] << 4) | full[:, 1::2]).astype(np.uint8).reshape(-1)
            got = codes.cpu().numpy()
            if not np.array_equal(got, packed):
                bad = int(np.flatnonzero(got != packed)[0])
                raise AssertionError(f"chunk {p0:#x} sign {sign}: first differing code byte {bad}")
            assert bool((absmax == 1.0).all())
    assert ops.device_error() == ops.QL_OK


def test_dequantize_ragged_sizes(ops):
    for nblocks in (1, 2, 5, 333):
        W = I.draw_w(I._streams(100 + nblocks), 1, 64 * nblocks, 0.5)
        check_roundtrip(ops, W)
