"""The seeded input generators: shapes, dtypes, ranges and determinism of the
recipes the oracle and the GPU path both consume."""
import numpy as np
import torch

from gated_delta_rule_98_b200 import synth


def test_draw_is_deterministic_and_shaped():
    a = synth.draw(70, 3, 32, 64, seed=5, dtype="bf16", num_seqs=2, s0_std=0.1)
    b = synth.draw(70, 3, 32, 64, seed=5, dtype="bf16", num_seqs=2, s0_std=0.1)
    for key in ("q", "k", "v", "z", "beta", "A", "S0"):
        assert torch.equal(a[key], b[key]), key
    assert a["q"].shape == (70, 3, 32) and a["v"].shape == (70, 3, 64)
    assert a["q"].dtype == torch.bfloat16 and a["A"].dtype == torch.float32
    assert a["S0"].shape == (2, 3, 32, 64) and a["S0"].dtype == torch.float32
    assert float(a["beta"].float().min()) > 0 and float(a["beta"].float().max()) < 1


def test_scalar_gate_range():
    g = synth.scalar_gate(4096, 4, seed=3)
    assert g.shape == (4096, 4) and g.dtype == torch.float32
    assert float(g.min()) >= -5.0 and float(g.max()) < 0.0
    assert torch.equal(g, synth.scalar_gate(4096, 4, seed=3))


def test_out_gate_and_conv_inputs():
    r, w = synth.out_gate_inputs(10, 2, 16, seed=1, dtype="f32")
    assert r.shape == (10, 2, 16) and r.dtype == torch.float32
    assert w.shape == (16,) and 0.5 <= float(w.min()) and float(w.max()) <= 1.5
    ci = synth.conv_inputs(12, 2, 8, 16, 3, seed=2)
    assert ci["x_q"].shape == (12, 2, 8) and ci["x_v"].shape == (12, 2, 16)
    assert ci["w_q"].shape == (16, 3) and ci["w_v"].shape == (32, 3)
    assert ci["x_k"].dtype == torch.bfloat16 and ci["w_k"].dtype == torch.float32


def test_varlen_lengths_recipe():
    lens = synth.varlen_lengths()
    assert sum(lens) == 32768 and all(512 <= L <= 8192 for L in lens)
    cu = synth.cu_from_lengths(lens)
    assert cu.dtype == torch.int32 and int(cu[-1]) == 32768
    assert np.all(np.diff(cu.numpy()) == np.array(lens))
