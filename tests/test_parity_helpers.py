"""The GPU parity checks themselves: a single wrong row must fail them even when the
aggregate error of the whole output is within the tolerance. CPU only."""

import numpy as np
import pytest
import torch

from parity import BF16_ROW_REL_L2, assert_bf16_parity, rel_l2, worst_row


def _pair(seed=0):
    r = np.random.default_rng(seed)
    ref = r.standard_normal((2, 4, 300, 64))
    got = ref * (1 + 1e-3 * r.standard_normal(ref.shape))   # bf16-sized noise everywhere
    return got, ref


def test_noise_at_bf16_level_passes():
    got, ref = _pair()
    assert_bf16_parity(torch.from_numpy(got), ref, 2, "noise")


def test_one_wrong_row_fails_although_the_aggregate_passes():
    got, ref = _pair(1)
    got[1, 3, 299] *= 1.1                    # the last row of a ragged tail off by 10%
    assert rel_l2(got, ref) < 5e-3            # invisible in the aggregate
    e, i = worst_row(got, ref)
    assert e > BF16_ROW_REL_L2 and i == (1 * 4 + 3) * 300 + 299
    with pytest.raises(AssertionError):
        assert_bf16_parity(torch.from_numpy(got), ref, 2, "planted row")


def test_a_fully_masked_row_must_be_exactly_zero():
    got, ref = _pair(2)
    ref[0, 0, 5] = 0.0
    got[0, 0, 5] = 0.0
    assert worst_row(got, ref)[0] < BF16_ROW_REL_L2
    got[0, 0, 5, 0] = 1e-3
    assert worst_row(got, ref)[0] == np.inf
