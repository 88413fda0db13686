"""kda_forward_checkpoints: the state after every `interval` tokens of each
sequence, compared with the float64 oracle's final state of the same inputs
cut after that many tokens (the oracle's final state is pinned elsewhere), on
the segmented tensor-core path, the unsegmented one, packed variable-length
sequences and the fp32 CUDA-core path.  Entries past a sequence's end must stay
untouched.  o and S_final must still match kda_forward's bar."""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import (TOL_BF16_ABS, TOL_BF16_REL, TOL_F32_ABS, assert_close, f64,
                          max_len_of, oracle_forward, rel_l2, to_cuda)

pytestmark = pytest.mark.gpu


def _bounds(inp):
    cu = inp.get("cu_seqlens")
    T, N = inp["q"].shape[0], inp["num_seqs"]
    return cu.numpy() if cu is not None else np.arange(N + 1) * (T // N if N else 0)


def _prefix(inp, E):
    """The inputs with every sequence cut after its first E tokens."""
    bnd = _bounds(inp)
    idx = np.concatenate([np.arange(bnd[n], min(bnd[n + 1], bnd[n] + E))
                          for n in range(len(bnd) - 1)]).astype(np.int64)
    out = {key: (val[idx] if key in ("q", "k", "v", "z", "beta") else val)
           for key, val in inp.items()}
    lens = [min(int(bnd[n + 1] - bnd[n]), E) for n in range(len(bnd) - 1)]
    out["cu_seqlens"] = synth.cu_from_lengths(lens)
    return out


def _check(inp, interval, chunk):
    bnd = _bounds(inp)
    N, H = inp["num_seqs"], inp["q"].shape[1]
    dk, dv = inp["q"].shape[2], inp["v"].shape[2]
    L = max_len_of(inp)
    J = L // interval
    d = to_cuda(inp)
    ck = torch.full((N, H, J, dk, dv), float("nan"), device="cuda")
    o, S, ck = kda.forward_checkpoints(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"],
                                       interval, S0=d.get("S0"), cu_seqlens=d.get("cu_seqlens"),
                                       num_seqs=N, max_seqlen=L, chunk=chunk, S_ckpt=ck)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, d["q"].dtype, "o")
    assert_close(S, S_ref, d["q"].dtype, "S_final")
    got = f64(ck)
    for j in range(J):
        E = (j + 1) * interval
        _, S_pre = oracle_forward(_prefix(inp, E))
        for n in range(N):
            if E <= bnd[n + 1] - bnd[n]:
                g, w = got[n, :, j], S_pre[n]
                err = np.abs(g - w).max()
                if d["q"].dtype == torch.float32:
                    assert err <= TOL_F32_ABS, (n, j, err)
                else:
                    assert err <= TOL_BF16_ABS and rel_l2(g, w) <= TOL_BF16_REL, (n, j, err)
            else:
                assert np.all(np.isnan(got[n, :, j])), f"entry ({n}, {j}) past the end was written"


def test_checkpoints_segmented_tensor_core_path():
    # one sequence, 4 heads: 8 segments per head (transition + chain passes)
    inp = synth.draw(1024, 4, 128, 128, seed=41, dtype="bf16", num_seqs=1, s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = None, 1
    _check(inp, 128, 64)


def test_checkpoints_unsegmented_tensor_core_path():
    # 8 sequences x 16 heads fill the GPU: one fused pass per (sequence, head)
    inp = synth.draw(8 * 128, 16, 128, 128, seed=42, dtype="bf16", num_seqs=8)
    inp["cu_seqlens"], inp["num_seqs"] = None, 8
    _check(inp, 64, 64)


def test_checkpoints_varlen_partial_and_empty_sequences():
    lens = [300, 64, 0, 411]
    inp = synth.draw(sum(lens), 4, 128, 128, seed=43, dtype="bf16", num_seqs=len(lens),
                     s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _check(inp, 128, 64)


def test_checkpoints_fp32_cuda_core_path():
    lens = [70, 33, 64]
    inp = synth.draw(sum(lens), 2, 32, 32, seed=44, dtype="f32", num_seqs=len(lens),
                     s0_std=0.1)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _check(inp, 32, 16)


def test_checkpoints_long_workload_full_size():
    """B=1, H=16, L=65536 (the long workload's launch configuration),
    checkpoints every 16384 tokens: the last one is the call's final state
    (the same fp32 values), and each earlier one matches the final state of a
    kda_forward call on that prefix within the bf16 bar (a different
    segmentation, so different bf16 rounding on the way)."""
    inp = synth.workload("long")
    d = to_cuda(inp)
    T = inp["q"].shape[0]
    o, S, ck = kda.forward_checkpoints(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], 16384,
                                       num_seqs=1, max_seqlen=T)
    o_plain, S_plain = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], num_seqs=1)
    torch.cuda.synchronize()
    assert torch.equal(o, o_plain) and torch.equal(S, S_plain)
    assert torch.equal(ck[:, :, 3], S)
    for j in range(3):
        E = 16384 * (j + 1)
        _, S_pre = kda.forward(d["q"][:E], d["k"][:E], d["v"][:E], d["z"][:E], d["A"],
                               d["beta"][:E], num_seqs=1)
        torch.cuda.synchronize()
        assert_close(ck[:, :, j], f64(S_pre), torch.bfloat16, f"checkpoint {j}")
