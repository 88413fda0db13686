"""Output epilogue (head-wise RMSNorm, gain, sigmoid output gate) fused into
the kernels that write o: kda_forward_norm_gate and kda_decode_step_norm_gate
against the float64 oracle (the recurrence, then ``oracle.epilogue``) on the
segmented and unsegmented tensor-core paths, packed sequences with a ragged
tail and an empty sequence, the CUDA-core path in fp32 and bf16, and the decode
step; at the long workload's full size, sampled rows against the oracle
epilogue applied to kda_forward's own o; gate extremes."""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, f64, max_len_of, oracle_forward, to_cuda

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _run(inp, chunk, weight=True, seed=7):
    from oracle import epilogue
    T, H, _ = inp["q"].shape
    dv = inp["v"].shape[2]
    r, w = synth.out_gate_inputs(T, H, dv, seed=seed, dtype=inp["q"].dtype)
    w = w if weight else None
    d = to_cuda(inp)
    y, S = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], r.cuda(),
                                 norm_weight=None if w is None else w.cuda(), eps=EPS,
                                 S0=d.get("S0"), cu_seqlens=d.get("cu_seqlens"),
                                 num_seqs=inp["num_seqs"], max_seqlen=max_len_of(inp),
                                 chunk=chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_forward(inp)
    y_ref = epilogue.norm_gate(o_ref, r, w, eps=EPS)
    assert_close(y, y_ref, inp["q"].dtype, "o (epilogue)")
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
    from oracle import epilogue, ref
    B, H = 6, 3
    inp = synth.draw(B, H, dk, dv, seed=55 + dk, dtype=dtype, num_seqs=B, s0_std=0.2)
    r, w = synth.out_gate_inputs(B, H, dv, seed=56, dtype=dtype)
    S = inp["S0"].cuda()
    y = kda.decode_step_norm_gate(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(),
                                  inp["z"].cuda(), inp["A"].cuda(), inp["beta"].cuda(), S,
                                  r.cuda(), norm_weight=w.cuda(), eps=EPS)
    torch.cuda.synchronize()
    o_ref, S_ref = ref.decode_step(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"],
                                   z=inp["z"], A=inp["A"])
    dt = inp["q"].dtype
    assert_close(y, epilogue.norm_gate(o_ref, r, w, eps=EPS), dt, "o (epilogue)")
    assert_close(S, S_ref, dt, "S")


def test_norm_gate_gate_extremes():
    """A closed gate writes zeros; a wide-open gate with unit gain leaves every
    (token, head) row with unit root mean square; the state is unaffected."""
    inp = synth.draw(8 * 128, 16, 128, 128, seed=57, dtype="bf16", num_seqs=8)
    d = to_cuda(inp)
    kw = dict(num_seqs=8, max_seqlen=128, chunk=64)
    o, S = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], **kw)
    closed = torch.full_like(d["v"], -100.0)
    y0, S0 = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], closed,
                                   **kw)
    y1, _ = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"],
                                  -closed, **kw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y0).item() == 0
    assert torch.equal(S0, S)
    rms = f64(y1).reshape(-1, 128)
    rms = np.sqrt(np.mean(rms * rms, axis=1))
    assert np.abs(rms - 1.0).max() < 1e-2


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
    assert_close(y[tt, ht], want, torch.bfloat16, "o (epilogue) sampled")
