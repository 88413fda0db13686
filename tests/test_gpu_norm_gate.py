"""Output epilogue (head-wise RMSNorm, gain, sigmoid output gate) fused into
the kernels that write o: kda_forward_norm_gate and kda_decode_step_norm_gate
on the segmented and unsegmented tensor-core paths, packed sequences with a
ragged tail and an empty sequence, the CUDA-core path in fp32 and bf16, and
the decode step; at the long workload's full size, sampled rows; gate
extremes.

Bars (derived from the arithmetic):
  (a) the fused epilogue against the float64 epilogue (``oracle.epilogue``)
      of the operator's own o from kda_forward on the same inputs: at most two
      roundings to the storage type apart (the staged o and y), so
      |dy| <= 2^-7 (|y| + 1) in bf16 and 1e-5 (|y| + 1) in fp32;
  (b) that o against the float64 oracle at the operator's own bar;
  (c) y against the oracle recurrence followed by the oracle epilogue: fp32
      max-abs 1e-4; bf16 relative L2 1e-2.  RMSNorm removes each row's scale,
      so a row's relative error in o becomes its absolute error in y, and the
      bf16 operator bar (absolute 2e-2, aggregate relative 5e-3) does not bound
      the relative error of rows whose norm is far below the typical one (the
      tensor-core path rounds the state and operands to bf16; about 9% of rows
      exceed 1% relative error, the worst ~50%, all of them rows of small norm).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import (TOL_F32_ABS, assert_close, f64, max_len_of, oracle_forward, rel_l2,
                          to_cuda)

pytestmark = pytest.mark.gpu

EPS = 1e-6
TOL_Y_BF16_REL = 1e-2


def _check(y, o_own, o_ref, r, w, dtype):
    from oracle import epilogue
    yg = f64(y)
    assert np.all(np.isfinite(yg))
    y_own = epilogue.norm_gate(f64(o_own), r, w, eps=EPS)
    tol = (2.0 ** -7 if dtype == torch.bfloat16 else 1e-5) * (np.abs(y_own) + 1.0)
    bad = np.abs(yg - y_own) > tol
    assert not bad.any(), f"(a) {bad.sum()} elements off the epilogue of the operator's o"
    assert_close(o_own, o_ref, dtype, "(b) o")
    y_ref = epilogue.norm_gate(o_ref, r, w, eps=EPS)
    if dtype == torch.float32:
        assert np.abs(yg - y_ref).max() <= TOL_F32_ABS
    else:
        assert rel_l2(yg, y_ref) <= TOL_Y_BF16_REL, rel_l2(yg, y_ref)


def _run(inp, chunk, weight=True, seed=7):
    T, H, _ = inp["q"].shape
    dv = inp["v"].shape[2]
    r, w = synth.out_gate_inputs(T, H, dv, seed=seed, dtype=inp["q"].dtype)
    w = w if weight else None
    d = to_cuda(inp)
    kw = dict(S0=d.get("S0"), cu_seqlens=d.get("cu_seqlens"), num_seqs=inp["num_seqs"],
              max_seqlen=max_len_of(inp), chunk=chunk)
    y, S = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], r.cuda(),
                                 norm_weight=None if w is None else w.cuda(), eps=EPS, **kw)
    o, S2 = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(S, S2)
    o_ref, S_ref = oracle_forward(inp)
    _check(y, o, o_ref, r, w, inp["q"].dtype)
    assert_close(S, S_ref, inp["q"].dtype, "S_final")


def test_norm_gate_segmented_tensor_core_path():
    inp = synth.draw(1024, 4, 128, 128, seed=51, dtype="bf16", num_seqs=1, s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = None, 1
    _run(inp, 64)


def test_norm_gate_unsegmented_tensor_core_path():
    inp = synth.draw(8 * 192, 16, 128, 128, seed=52, dtype="bf16", num_seqs=8)
    inp["cu_seqlens"], inp["num_seqs"] = None, 8
    _run(inp, 64)


def test_norm_gate_varlen_ragged_and_empty():
    lens = [300, 64, 0, 411, 1]
    inp = synth.draw(sum(lens), 4, 128, 128, seed=53, dtype="bf16", num_seqs=len(lens),
                     s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _run(inp, 64, weight=False)


@pytest.mark.parametrize("dtype,chunk,d", [("f32", 16, 64), ("f32", 64, 32), ("bf16", 64, 64)])
def test_norm_gate_cuda_core_path(dtype, chunk, d):
    lens = [70, 33, 130]
    inp = synth.draw(sum(lens), 2, d, d, seed=54, dtype=dtype, num_seqs=len(lens), s0_std=0.1)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _run(inp, chunk)


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "bf16"), (32, 32, "f32"), (64, 128, "f32")])
def test_decode_norm_gate(dk, dv, dtype):
    from oracle import ref
    B, H = 6, 3
    inp = synth.draw(B, H, dk, dv, seed=55 + dk, dtype=dtype, num_seqs=B, s0_std=0.2)
    r, w = synth.out_gate_inputs(B, H, dv, seed=56, dtype=dtype)
    args = [inp[n].cuda() for n in ("q", "k", "v", "z", "A", "beta")]
    S = inp["S0"].cuda()
    S_plain = S.clone()
    y = kda.decode_step_norm_gate(*args, S, r.cuda(), norm_weight=w.cuda(), eps=EPS)
    o = kda.decode_step(*args, S_plain)
    torch.cuda.synchronize()
    assert torch.equal(S, S_plain)
    o_ref, S_ref = ref.decode_step(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"],
                                   z=inp["z"], A=inp["A"])
    _check(y, o, o_ref, r, w, inp["q"].dtype)
    assert_close(S, S_ref, inp["q"].dtype, "S")


def test_norm_gate_gate_extremes():
    """A closed gate writes zeros; a wide-open gate with unit gain leaves every
    (token, head) row with root mean square sqrt(ms / (ms + eps)), ms the mean
    square of the operator's o in that row; the state is unaffected."""
    inp = synth.draw(8 * 128, 16, 128, 128, seed=57, dtype="bf16", num_seqs=8)
    d = to_cuda(inp)
    kw = dict(num_seqs=8, max_seqlen=128, chunk=64)
    o, S = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], **kw)
    closed = torch.full_like(d["v"], -100.0)
    y0, S0 = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], closed,
                                   eps=EPS, **kw)
    y1, _ = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"],
                                  -closed, eps=EPS, **kw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y0).item() == 0
    assert torch.equal(S0, S)
    y1 = f64(y1).reshape(-1, 128)
    ms = np.mean(f64(o).reshape(-1, 128) ** 2, axis=1)
    want = np.sqrt(ms / (ms + EPS))
    assert np.abs(np.sqrt(np.mean(y1 * y1, axis=1)) - want).max() < 1e-2


def test_norm_gate_long_workload_sampled():
    """B=1, H=16, L=65536 (the long workload's launch configuration): sampled
    rows of the fused epilogue against the float64 epilogue of kda_forward's o
    (whose parity with the oracle is tested at this size elsewhere)."""
    from oracle import epilogue
    inp = synth.workload("long")
    d = to_cuda(inp)
    T, H, _ = inp["q"].shape
    r, w = synth.out_gate_inputs(T, H, 128, seed=58)
    rc, wc = r.cuda(), w.cuda()
    kw = dict(num_seqs=1, max_seqlen=T, chunk=64)
    o, S = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], **kw)
    y, Sy = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], rc,
                                  norm_weight=wc, eps=EPS, **kw)
    torch.cuda.synchronize()
    assert torch.equal(S, Sy)
    rng = np.random.default_rng(59)
    ts = np.concatenate([rng.choice(T, 2048, replace=False), [0, 63, 64, T - 1]])
    hs = rng.integers(0, H, ts.size)
    tt, ht = torch.from_numpy(ts).cuda(), torch.from_numpy(hs).cuda()
    want = epilogue.norm_gate(f64(o[tt, ht]), r[ts, hs], w, eps=EPS)
    got = f64(y[tt, ht])
    assert np.all(np.abs(got - want) <= 2.0 ** -7 * (np.abs(want) + 1.0))
