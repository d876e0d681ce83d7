"""GPU parity of qlora_linear_fwd / qlora_linear_bwd against the fp64 oracle, through the C ABI.

Tolerance (stated for the layer): relative Frobenius error <= 1e-2 and max-abs error <= 2e-2 * max|ref|,
against the oracle evaluated in fp64 on the same host inputs.  Small shapes span several tiles and a
ragged tail in every dimension; the full workloads run in the launch configuration the benchmark times
and are compared on sampled token rows (every output row is independent of the others) plus the full
rank-r gradients.
"""

import numpy as np
import pytest
import torch

from oracle import linear as L
from oracle import nf4 as O
from qlora_fine_tuning_blockwise_b200 import inputs as I
from tests.gpu_common import assert_close, dev, f64, lora_or_none, oracle_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def run_gpu(ops, d, need_bwd=True, pass_su=True):
    N, K, r, s = d["N"], d["K"], d["r"], d["s"]
    codes, absmax = ops.nf4_quantize(dev(d["W"]))
    x = dev(d["x"])
    A, B = lora_or_none(d)
    y, su = ops.qlora_linear_fwd(x, codes, absmax, A, B, s, N, K)
    out = dict(y=y, su=su)
    if need_bwd:
        dy = dev(d["dy"])
        dx, dA, dB = ops.qlora_linear_bwd(dy, x, codes, absmax, A, B, s, N, K, su=su if pass_su else None)
        out.update(dx=dx, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert ops.device_error() == ops.QL_OK
    return out


def oracle_all(d, rows=None):
    """Oracle outputs from the host inputs; with ``rows`` the row-wise outputs only at those token rows."""
    Wd = oracle_weight(d["W"])
    x, A, B, dy, s = f64(d["x"]), f64(d["A"]), f64(d["B"]), f64(d["dy"]), d["s"]
    xs = x if rows is None else x[rows]
    dys = dy if rows is None else dy[rows]
    ref = dict(y=L.qlora_forward(xs, Wd, A, B, s), su=s * L.lora_down(xs, A))
    if rows is None:
        ref["dx"], ref["dA"], ref["dB"] = L.qlora_backward(dy, x, Wd, A, B, s)
    else:
        ref["dx"] = L.qlora_backward(dys, xs, Wd, A, B, s)[0]
        ref["dA"], ref["dB"] = L.lora_grads(dy, x, A, B, s)
    return ref


SMALL = [
    # M, N, K, r
    (64, 256, 256, 8),      # the tiny workload's shape
    (1, 264, 192, 16),      # one token; ragged N tile
    (17, 136, 320, 72),     # r spans two 64-wide extra stages
    (130, 8, 64, 0),        # plain NF4 layer, N smaller than a tile
    (300, 264, 256, 16),    # ragged token tiles at BN = 256
    (257, 512, 640, 64),
    (33, 1024, 1984, 8),    # K % 128 == 64: half-empty transposed tile in dX
    (520, 128, 128, 256),   # largest rank
    # token-light layers with K % 256 == 0 run the forward in stages of four NF4 blocks
    (1, 264, 512, 16),      # BN = 16, ragged N tile
    (40, 136, 768, 72),     # BN = 64, odd number of 4-block stages, partly filled LoRA stage
    (20, 128, 1280, 256),   # BN = 32, largest rank in one 256-wide LoRA stage
    # token-light layers deep enough for the stream-K schedule (tiles shared by consecutive CTAs, fp32 slabs)
    (16, 1024, 4096, 16),   # 4-block stages, four CTAs per tile
    (40, 2056, 2048, 72),   # BN = 64, ragged weight tile, two CTAs per tile
    (8, 1024, 2112, 8),     # K % 256 != 0: one-block stages
]


@pytest.mark.parametrize("M,N,K,r", SMALL)
def test_forward_backward_small(ops, M, N, K, r):
    d = I.make_random_linear(M, N, K, r, s=2.0, seed=M + N + K + r)
    got = run_gpu(ops, d)
    ref = oracle_all(d)
    assert_close(got["y"], ref["y"], "y")
    assert_close(got["dx"], ref["dx"], "dX")
    if r:
        assert_close(got["su"], ref["su"], "s*x*A^T")
        assert_close(got["dA"], ref["dA"], "dA")
        assert_close(got["dB"], ref["dB"], "dB")


@pytest.mark.parametrize("M,N,K,r,s", [
    (64, 256, 256, 8, -1.5),     # BN = 64 forward, one LoRA stage
    (300, 264, 256, 16, -2.0),   # BN = 256 forward, ragged token and weight tiles
    (1, 264, 512, 16, -0.25),    # token-light forward in four-block stages
    (40, 136, 768, 72, -1.0),    # two LoRA stages, partly filled
])
def test_negative_scaling(ops, M, N, K, r, s):
    """A negative s flips the sign of the LoRA term in y, of v = s dY B in dX and of both adapter gradients."""
    d = I.make_random_linear(M, N, K, r, s=s, seed=M + N + K + r + 1000)
    got = run_gpu(ops, d)
    ref = oracle_all(d)
    for k, name in (("y", "y"), ("dx", "dX"), ("su", "s*x*A^T"), ("dA", "dA"), ("dB", "dB")):
        assert_close(got[k], ref[k], f"{name} s={s}")
    # the LoRA term really is subtracted: removing it moves y away from the reference
    base = L.qlora_forward(f64(d["x"]), oracle_weight(d["W"]), f64(d["A"]), f64(d["B"]), 0.0)
    assert np.linalg.norm(base - ref["y"]) > 1e-2 * np.linalg.norm(ref["y"])


def test_backward_recomputes_su_when_not_given(ops):
    d = I.make_random_linear(96, 264, 320, 16, s=0.5, seed=11)
    a = run_gpu(ops, d, pass_su=True)
    b = run_gpu(ops, d, pass_su=False)
    for k in ("dx", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k


def test_tiny_workload_full(ops):
    d = I.make_linear_inputs("tiny_64x256x256_r8")
    got = run_gpu(ops, d)
    ref = oracle_all(d)
    for k in ("y", "su", "dx", "dA", "dB"):
        assert_close(got[k], ref[k], k)


@pytest.mark.parametrize("M", [200, 16])
def test_B_zero_equals_plain_layer_bitwise(ops, M):
    """B = 0 appends products that are all zero: y must equal the r = 0 layer bit for bit (M = 16 takes the
    4-block stages of the token-light forward)."""
    d = I.make_random_linear(M, 384, 512, 16, seed=5)
    codes, absmax = ops.nf4_quantize(dev(d["W"]))
    x = dev(d["x"])
    A = dev(d["A"])
    B0 = torch.zeros(384, 16, dtype=torch.bfloat16, device="cuda")
    y_b0, _ = ops.qlora_linear_fwd(x, codes, absmax, A, B0, 2.0, 384, 512)
    y_r0, _ = ops.qlora_linear_fwd(x, codes, absmax, None, None, 2.0, 384, 512)
    assert torch.equal(y_b0, y_r0)
    ref = f64(d["x"]) @ oracle_weight(d["W"]).T
    assert_close(y_r0, ref, "base layer")


def test_s_zero_and_A_zero(ops):
    d = I.make_random_linear(64, 256, 256, 8, seed=6)
    codes, absmax = ops.nf4_quantize(dev(d["W"]))
    x, dy = dev(d["x"]), dev(d["dy"])
    A, B = dev(d["A"]), dev(d["B"])
    y_s0, _ = ops.qlora_linear_fwd(x, codes, absmax, A, B, 0.0, 256, 256)
    y_r0, _ = ops.qlora_linear_fwd(x, codes, absmax, None, None, 0.0, 256, 256)
    assert torch.equal(y_s0, y_r0)
    A0 = torch.zeros_like(A)
    dx, dA, dB = ops.qlora_linear_bwd(dy, x, codes, absmax, A0, B, 2.0, 256, 256)
    assert torch.count_nonzero(dB) == 0
    dx0, _, _ = ops.qlora_linear_bwd(dy, x, codes, absmax, None, None, 2.0, 256, 256)
    assert torch.equal(dx, dx0)


def test_empty_batch(ops):
    d = I.make_random_linear(4, 256, 256, 8, seed=7)
    codes, absmax = ops.nf4_quantize(dev(d["W"]))
    A, B = dev(d["A"]), dev(d["B"])
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    y, su = ops.qlora_linear_fwd(x, codes, absmax, A, B, 2.0, 256, 256)
    assert y.shape == (0, 256)
    dA = torch.full((8, 256), 7.0, device="cuda")
    dB = torch.full((256, 8), 7.0, device="cuda")
    _, dA, dB = ops.qlora_linear_bwd(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), x, codes, absmax, A, B,
                                     2.0, 256, 256, need_dx=False, dA=dA, dB=dB)
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


def test_deterministic(ops):
    d = I.make_random_linear(600, 512, 1024, 16, seed=8)
    a = run_gpu(ops, d)
    b = run_gpu(ops, d)
    for k in ("y", "su", "dx", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("name", ["attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64"])
def test_workload_full_size_sampled_rows(ops, name):
    d = I.make_linear_inputs(name)
    got = run_gpu(ops, d)
    rows = np.sort(np.random.default_rng(1).choice(d["M"], size=64, replace=False))
    ref = oracle_all(d, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    assert_close(got["y"][idx], ref["y"], "y rows")
    assert_close(got["su"][idx], ref["su"], "su rows")
    assert_close(got["dx"][idx], ref["dx"], "dX rows")
    assert_close(got["dA"], ref["dA"], "dA")
    assert_close(got["dB"], ref["dB"], "dB")


@pytest.mark.parametrize("name", ["attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64"])
def test_workload_full_size_repeatable(ops, name):
    """Every reduction runs in a fixed order, so repeated passes must agree bit for bit; a race between the
    kernel's warp roles (a slot refilled or overwritten too early) shows up here as a mismatch."""
    d = I.make_linear_inputs(name)
    layer = ops.QLoRALinear(dev(d["W"]), dev(d["A"]), dev(d["B"]), d["s"])
    x, dy = dev(d["x"]), dev(d["dy"])
    first = None
    for _ in range(4):
        y, su = layer.forward(x)
        dx, dA, dB = layer.backward(dy, x, su=su)
        torch.cuda.synchronize()
        outs = [t.clone() for t in (y, dx, dA, dB)]
        if first is None:
            first = outs
        else:
            for what, a, b in zip(("y", "dX", "dA", "dB"), first, outs):
                assert torch.equal(a, b), f"{what} differs between repeated passes"
    assert ops.device_error() == ops.QL_OK


def test_decode_workload_full_size_sampled_columns(ops):
    """16 tokens x 28672 outputs: every output column n needs only weight row n, so the oracle quantizes a
    random sample of 512 rows of W and checks those columns of y for all 16 tokens."""
    d = I.make_linear_inputs("decode_16x8192x28672_r16")
    got = run_gpu(ops, d, need_bwd=False)
    cols = np.sort(np.random.default_rng(2).choice(d["N"], size=512, replace=False))
    Wd = oracle_weight(d["W"][cols])
    ref = L.qlora_forward(f64(d["x"]), Wd, f64(d["A"]), f64(d["B"])[cols], d["s"])
    assert_close(got["y"][:, torch.from_numpy(cols).cuda()], ref, "y columns")
