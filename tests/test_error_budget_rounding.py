"""The rounding helpers of tests/error_budget.py against torch's own
conversions (CPU): the error budget is only as good as its emulated bf16,
f16 and tf32 roundings."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import error_budget as eb  # noqa: E402


def _samples():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, -1.0, 1.00390625, 1.0078125, 3.0e38, -3.0e38, 1e-40]])
    return x.astype(np.float32)


def test_bf16_matches_torch():
    x = _samples()
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(eb.bf16(x), want)


def test_f16_matches_torch_in_range():
    x = _samples()
    x = x[np.abs(x) <= 65504]
    want = torch.from_numpy(x).to(torch.float16).float().numpy()
    assert np.array_equal(eb.f16(x), want)


def test_tf32_keeps_ten_mantissa_bits():
    x = _samples()
    x = x[(np.abs(x) > 1e-30) & (np.abs(x) < 1e30)]
    y = eb.tf32(x)
    assert np.all(np.abs(y - x) <= np.abs(x) * 2.0 ** -11)
    # the 13 low mantissa bits are clear
    assert np.all((y.view(np.uint32) & 0x1FFF) == 0)


def test_hi_lo_pair_is_near_float32():
    x = _samples()
    x = x[(np.abs(x) > 1e-30) & (np.abs(x) < 1e30)]
    y = eb.hi_lo(x)
    assert np.all(np.abs(y - x) <= np.abs(x) * 2.0 ** -16)
