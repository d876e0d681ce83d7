"""The bounded chain sample (used by the benchmark's CPU baseline and reference arm) is an exact slice of the full
chain's draws: its first m tokens and first f intermediate features."""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_blockwise_b200 import inputs as I


def test_chain_sample_is_a_slice_of_the_full_draws():
    full = I.make_chain_inputs(M=40, D=128, F=512, r=8)
    smp = I.make_chain_sample(16, 192, D=128, F=512, r=8)
    assert torch.equal(smp["x"], full["x"][:16]) and torch.equal(smp["dy"], full["dy"][:16])
    for n in ("gate", "up"):
        assert np.array_equal(smp["layers"][n]["W"], full["layers"][n]["W"][:192])
        assert torch.equal(smp["layers"][n]["A"], full["layers"][n]["A"])
        assert torch.equal(smp["layers"][n]["B"], full["layers"][n]["B"][:192])
    assert np.array_equal(smp["layers"]["down"]["W"], full["layers"]["down"]["W"][:, :192])
    assert torch.equal(smp["layers"]["down"]["A"], full["layers"]["down"]["A"][:, :192])
    assert torch.equal(smp["layers"]["down"]["B"], full["layers"]["down"]["B"])
    assert smp["F"] == 192 and smp["M"] == 16


def test_chain_sample_rejects_partial_blocks():
    with pytest.raises(ValueError):
        I.make_chain_sample(8, 100, D=128, F=512, r=8)
