"""The error-budget script (tests/error_budget.py) pinned on the CPU: its
bf16, f16 and tf32 roundings against torch's own conversions, and its
chunkwise algebra, with every rounding off, against the float64 oracle.  The
budget is only as good as these two."""
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


def test_emulation_without_rounding_is_the_oracle():
    """With every rounding off, the emulated chunkwise form (both chain
    schedules, 64- and 128-token chunks) agrees with the float64 oracle to
    float32 accuracy, so the budget measures roundings and nothing else."""
    from gated_delta_rule_98_b200 import synth
    from oracle import ref
    inp = synth.draw(512, 2, 128, 128, seed=9, dtype="bf16")
    d = {n: inp[n].double().numpy() for n in ("q", "k", "v", "beta", "z")}
    o_ref, _ = ref.forward(d["q"], d["k"], d["v"], d["beta"], z=d["z"],
                           A=inp["A"].double().numpy())
    for kw in (dict(), dict(reassociated=True), dict(C=128)):
        o = eb.chunked(inp, [0, 1], eb.NONE, **kw)
        assert np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref) < 1e-5, kw
