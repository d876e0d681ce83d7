"""Pins for the NF4 oracle (``oracle.nf4``) against what the mathematics fixes, independent of the oracle.

Each test would fail on a plausible mistake in the oracle: a wrong quantile, a mis-normalised table, a
lost level, ties broken upward, a swapped nibble order, a scale applied twice, a double rounding.
"""

import math
from statistics import NormalDist

import numpy as np
import pytest
import scipy.special
import torch

from oracle import nf4 as O
from qlora_fine_tuning_blockwise_b200 import inputs as I


def f32_ulp(x: float) -> float:
    x = np.float32(abs(x))
    return float(np.nextafter(x, np.float32(np.inf)) - x)


# ---------------------------------------------------------------------------------------------- quantile


def test_normal_quantile_matches_library_routines():
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 401), [0.5, 0.9677083333333334, 0.75, 0.25, 1e-9]])
    for p in ps:
        z = O.normal_quantile(float(p))
        assert abs(z - scipy.special.ndtri(p)) <= 4e-15 * max(1.0, abs(z)), p
        assert abs(z - NormalDist().inv_cdf(float(p))) <= 4e-15 * max(1.0, abs(z)), p


def test_normal_quantile_closed_points():
    assert O.normal_quantile(0.5) == 0.0
    # Phi(1.959963984540054) = 0.975 to double precision (textbook 97.5% point)
    assert abs(O.normal_quantile(0.975) - 1.959963984540054) < 1e-14
    assert abs(O.normal_quantile(0.8413447460685429) - 1.0) < 1e-14  # Phi(1)
    with pytest.raises(ValueError):
        O.normal_quantile(1.0)


# ---------------------------------------------------------------------------------------------- codebook


def test_codebook_invariants():
    c = O.nf4_codebook()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.all(np.diff(c.astype(np.float64)) > 0)
    assert c[7] == 0.0 and not np.signbit(c[7])
    assert c[0] == -1.0 and c[15] == 1.0
    assert int(np.sum(c > 0)) == 8 and int(np.sum(c < 0)) == 7
    assert np.all(np.abs(c) <= 1.0)


def test_codebook_levels_are_normalised_quantiles_second_method():
    """Each level equals Phi^-1(p)/Phi^-1(1-delta) computed with an independent quantile routine."""
    c = O.nf4_codebook()
    delta = (1 / 32 + 1 / 30) / 2
    nd = NormalDist()
    top = nd.inv_cdf(1 - delta)
    pos = [nd.inv_cdf((1 - delta) + i * (0.5 - (1 - delta)) / 8) / top for i in range(8)]
    neg = [-nd.inv_cdf((1 - delta) + i * (0.5 - (1 - delta)) / 7) / top for i in range(7)]
    expect = sorted(pos + neg + [0.0])
    for got, want in zip(c, expect):
        assert abs(float(got) - want) <= f32_ulp(want), (got, want)
    # and the fp32 table is the single rounding of those values wherever the second method is not
    # within a hair of a rounding boundary
    exact = np.array(expect, dtype=np.float64).astype(np.float32)
    assert np.sum(exact != c) <= 1


def test_codebook_golden_fixture():
    """The stored table (written by tests/golden/make_golden.py from the oracle) is what the oracle builds."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nf4_codebook.txt")
    vals = []
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            idx, hexbits, dec = line.split()
            vals.append(np.uint32(int(hexbits, 16)).view(np.float32))
    assert np.array_equal(np.array(vals, dtype=np.float32).view(np.uint32), O.nf4_codebook().view(np.uint32))


def _paper_table() -> np.ndarray:
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nf4_qlora_paper.txt")
    vals = []
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            idx, dec = line.split()
            assert int(idx) == len(vals)
            vals.append(float(dec))
    assert len(vals) == 16
    return np.array(vals, dtype=np.float64)


def _paper_mismatch(table: np.ndarray) -> float:
    """Largest relative difference between a 16-level table and the printed NF4 values (absolute at 0)."""
    ref = _paper_table()
    t = np.asarray(table, dtype=np.float64)
    return float(np.max(np.abs(t - ref) / np.maximum(np.abs(ref), 1.0e-30 + (ref == 0))))


PAPER_RTOL = 1.0e-6  # the printed values are fp32 levels written out in decimal; the rule reproduces them


def test_codebook_matches_the_published_nf4_values():
    """The level set equals the 16 values printed in the QLoRA paper (Appendix E), the public definition of
    NF4 that reading R1 follows -- a pin from outside the oracle, not a restatement of its formula."""
    c = O.nf4_codebook()
    assert _paper_mismatch(c) <= PAPER_RTOL
    # within a few fp32 ulps of the printed values, level by level
    ref32 = _paper_table().astype(np.float32)
    assert np.max(np.abs(c.view(np.int32).astype(np.int64) - ref32.view(np.int32).astype(np.int64))) <= 8


@pytest.mark.parametrize("mistake", ["delta_1_32", "delta_1_30", "nine_point_negative_grid", "eight_point_positive_grid",
                                     "uniform_instead_of_normal_quantiles"])
def test_codebook_pin_catches_planted_mistakes(monkeypatch, mistake):
    """Each plausible slip in the construction moves some level by far more than the pin's tolerance."""
    if mistake == "delta_1_32":
        monkeypatch.setattr(O, "NF4_DELTA", 1.0 / 32.0)
    elif mistake == "delta_1_30":
        monkeypatch.setattr(O, "NF4_DELTA", 1.0 / 30.0)
    elif mistake == "uniform_instead_of_normal_quantiles":
        monkeypatch.setattr(O, "normal_quantile", lambda p: p - 0.5)
    else:
        top = 1.0 - O.NF4_DELTA

        def probs():
            npos, nneg = {"nine_point_negative_grid": (8, 8), "eight_point_positive_grid": (7, 7)}[mistake]
            pos = [top + i * (0.5 - top) / npos for i in range(8)]
            neg = [top + i * (0.5 - top) / nneg for i in range(7)]
            return pos, neg
        monkeypatch.setattr(O, "nf4_probabilities", probs)
    assert _paper_mismatch(O.nf4_codebook()) > 100 * PAPER_RTOL


# ---------------------------------------------------------------------------------------------- quantize


def argmin_code(n: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Independent nearest-level rule: argmin_i |n - c_i| (exact fp64 distances), ties to the lower index."""
    d = np.abs(n.astype(np.float64)[:, None] - c.astype(np.float64)[None, :])
    return np.argmin(d, axis=1).astype(np.uint8)  # argmin returns the first (lowest) index on ties


def _test_values():
    c = O.nf4_codebook()
    grid = np.linspace(-1, 1, 200001).astype(np.float32)
    mids = ((c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2)
    near = []
    for m in mids:
        f = np.float32(m)
        for k in range(-3, 4):
            v = f
            step = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
            for _ in range(abs(k)):
                v = np.nextafter(v, step)
            near.append(v)
    for lv in c:
        near += [np.nextafter(lv, np.float32(-2)), lv, np.nextafter(lv, np.float32(2))]
    vals = np.concatenate([grid, np.array(near, dtype=np.float32)])
    return vals[(vals >= -1) & (vals <= 1)]


def test_code_rule_matches_bruteforce_nearest_level():
    c = O.nf4_codebook()
    n = _test_values()
    assert np.array_equal(O.nf4_code_of(n), argmin_code(n, c))


def test_midpoint_ties_go_to_lower_code():
    c = O.nf4_codebook()
    mids = (c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2
    hit = 0
    for i, m in enumerate(mids):
        f = np.float32(m)
        if float(f) == m:  # the midpoint is itself an fp32 value: an exact tie
            hit += 1
            assert O.nf4_code_of(np.array([f]))[0] == i
            assert argmin_code(np.array([f]), c)[0] == i
    assert hit >= 1  # several midpoints of the fp32 table are themselves fp32 values


def test_tie_rule_on_a_table_with_exact_midpoints():
    """On a table of dyadic levels every midpoint is an fp32 value: each exact tie must take the lower code."""
    c = np.linspace(-1, 1, 16).astype(np.float64)
    c = np.round(c * 64) / 64
    c[7] = 0.0
    c = np.sort(c).astype(np.float32)
    mids = (c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2
    n = mids.astype(np.float32)
    assert np.array_equal(n.astype(np.float64), mids)
    assert np.array_equal(O.nf4_code_of(n, c), np.arange(15))
    assert np.array_equal(argmin_code(n, c), np.arange(15))


def test_worked_block_fixture():
    """tests/golden/nf4_worked_block.txt: w_j = c_(j mod 16) / 2, so absmax = 1/2 and code_j = j mod 16."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nf4_worked_block.txt")
    lines = [l.split("#")[0].strip() for l in open(path)]
    lines = [l for l in lines if l]
    absmax_hex = lines[0].split()[1]
    code_bytes = bytes.fromhex("".join(lines[1:]).replace("codes", "").replace(" ", ""))
    c = O.nf4_codebook()
    w = np.array([c[j % 16] / np.float32(2) for j in range(64)], dtype=np.float32)
    codes, absmax = O.nf4_quantize(w)
    assert absmax.view(np.uint32)[0] == int(absmax_hex, 16) == np.float32(0.5).view(np.uint32)
    assert codes.tobytes() == code_bytes
    assert code_bytes[:4] == bytes([0x01, 0x23, 0x45, 0x67])  # R5: element 2j in the high nibble


def test_packing_high_nibble_first():
    w = np.zeros(64, np.float32)
    w[0], w[1] = 3.0, -3.0          # n = +1 -> code 15, n = -1 -> code 0
    codes, absmax = O.nf4_quantize(w)
    assert absmax[0] == 3.0
    assert codes[0] == 0xF0 and codes[1] == 0x77 and np.all(codes[1:] == 0x77)
    assert np.array_equal(O.nf4_unpack(codes)[:4], [15, 0, 7, 7])


def test_zero_block():
    w = np.zeros(128, np.float32)
    w[64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    codes, absmax = O.nf4_quantize(w)
    assert absmax[0] == 0.0 and np.all(codes[:32] == 0x77)
    deq = O.nf4_dequantize(codes, absmax, 128)
    assert np.all(deq[:64] == 0.0)


def test_block_extreme_reproduces_absmax_exactly():
    w = I.draw_w(I._streams(5), 64, 512, 0.02).reshape(-1)
    codes, absmax = O.nf4_quantize(w)
    deq = O.nf4_dequantize(codes, absmax, w.size)
    blocks = w.reshape(-1, 64)
    dblocks = deq.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        j = int(np.argmax(np.abs(blocks[b])))
        assert dblocks[b, j] == blocks[b, j]  # +-1 level times absmax is exact


def test_scale_invariance_powers_of_two():
    w = I.draw_w(I._streams(6), 32, 256, 0.02).reshape(-1)
    codes0, absmax0 = O.nf4_quantize(w)
    for k in (-4, -1, 1, 3, 10):
        f = np.float32(2.0 ** k)
        codes, absmax = O.nf4_quantize(w * f)
        assert np.array_equal(codes, codes0)
        assert np.array_equal(absmax, absmax0 * f)


def test_error_bound_half_local_gap():
    c = O.nf4_codebook().astype(np.float64)
    w = I.draw_w(I._streams(7), 64, 1024, 0.02).reshape(-1)
    codes, absmax = O.nf4_quantize(w)
    deq = O.nf4_dequantize(codes, absmax, w.size).astype(np.float64)
    scale = np.repeat(absmax.astype(np.float64), 64)
    n = w.astype(np.float64) / scale
    i = np.clip(np.searchsorted(c, n, side="right") - 1, 0, 14)  # interval [c_i, c_{i+1}] holding n
    half_gap = (c[i + 1] - c[i]) / 2
    ulp = np.array([f32_ulp(a) for a in absmax]).repeat(64)
    assert np.all(np.abs(deq - w) <= half_gap * scale + 2 * ulp)


def test_nf4_beats_int4_on_normal_blocks():
    """NF4 has smaller quantization error than INT4 at the same width on normally distributed weights."""
    w = I.draw_w(I._streams(8), 256, 1024, 0.02).reshape(-1)
    codes, absmax = O.nf4_quantize(w)
    deq = O.nf4_dequantize(codes, absmax, w.size)
    blocks = w.reshape(-1, 64).astype(np.float64)
    am = np.abs(blocks).max(axis=1, keepdims=True)
    q = np.clip(np.rint(blocks / am * 7), -7, 7)
    int4 = (q / 7 * am).reshape(-1)
    rms_nf4 = np.sqrt(np.mean((deq - w) ** 2))
    rms_int4 = np.sqrt(np.mean((int4 - w) ** 2))
    assert rms_nf4 < rms_int4


def test_quotient_single_rounding_equals_ieee_fp32_division():
    rng = np.random.default_rng(3)
    a = rng.standard_normal(100000).astype(np.float32)
    b = np.abs(rng.standard_normal(100000).astype(np.float32)) + np.float32(1e-3)
    via64 = (a.astype(np.float64) / b.astype(np.float64)).astype(np.float32)
    t = (torch.from_numpy(a) / torch.from_numpy(b)).numpy()
    assert np.array_equal(via64.view(np.uint32), t.view(np.uint32))


def test_nonfinite_rejected():
    w = np.zeros(64, np.float32)
    w[3] = np.inf
    with pytest.raises(ValueError):
        O.nf4_quantize(w)


# ---------------------------------------------------------------------------------------------- dequantize


def test_dequantize_is_one_fp32_rounding_of_product():
    w = I.draw_w(I._streams(9), 16, 512, 0.02).reshape(-1)
    codes, absmax = O.nf4_quantize(w)
    deq = O.nf4_dequantize(codes, absmax, w.size)
    c = O.nf4_codebook()
    idx = O.nf4_unpack(codes)
    ref = (torch.from_numpy(c[idx]) * torch.from_numpy(np.repeat(absmax, 64))).numpy()  # IEEE fp32 multiply
    assert np.array_equal(deq.view(np.uint32), ref.view(np.uint32))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    a = np.concatenate([rng.standard_normal(200000).astype(np.float32) * np.float32(0.03),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1.5e-40, 1e-45], np.float32)])
    # include exact ties: patterns whose low 16 bits are 0x8000
    ties = (rng.integers(0, 2 ** 31, 1000, dtype=np.uint64).astype(np.uint32) & np.uint32(0x7F7F0000)) | np.uint32(0x8000)
    a = np.concatenate([a, ties.view(np.float32)])
    ours = O.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
