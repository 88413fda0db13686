"""kda_forward_scalar_gate (the Gated DeltaNet case: one log-decay per token
and head, shared by the channels) against the float64 oracle run with that
gate broadcast over the dk channels, on the segmented and unsegmented
tensor-core paths, packed sequences with a ragged tail and an empty sequence,
and the CUDA-core path; and against kda_forward_g given the broadcast gate,
which must agree exactly (same arithmetic, z not read)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, max_len_of, oracle_forward, to_cuda

pytestmark = pytest.mark.gpu


def _run(inp, chunk, seed):
    T, H, dk = inp["q"].shape
    gs = synth.scalar_gate(T, H, seed=seed)
    g_full = gs[:, :, None].expand(T, H, dk).contiguous()
    d = to_cuda(inp)
    kw = dict(S0=d.get("S0"), cu_seqlens=d.get("cu_seqlens"), num_seqs=inp["num_seqs"],
              max_seqlen=max_len_of(inp), chunk=chunk)
    o, S = kda.forward_scalar_gate(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], **kw)
    og, Sg = kda.forward_g(d["q"], d["k"], d["v"], g_full.cuda(), d["beta"], **kw)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_forward(inp, g=g_full)
    assert_close(o, o_ref, inp["q"].dtype, "o")
    assert_close(S, S_ref, inp["q"].dtype, "S_final")
    assert torch.equal(o, og) and torch.equal(S, Sg)


def test_scalar_gate_segmented_tensor_core_path():
    inp = synth.draw(1024, 4, 128, 128, seed=61, dtype="bf16", num_seqs=1, s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = None, 1
    _run(inp, 64, 1)


def test_scalar_gate_unsegmented_tensor_core_path():
    inp = synth.draw(8 * 192, 16, 128, 128, seed=62, dtype="bf16", num_seqs=8)
    inp["cu_seqlens"], inp["num_seqs"] = None, 8
    _run(inp, 64, 2)


def test_scalar_gate_varlen_ragged_and_empty():
    lens = [300, 0, 411, 17]
    inp = synth.draw(sum(lens), 4, 128, 128, seed=63, dtype="bf16", num_seqs=len(lens),
                     s0_std=0.02)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _run(inp, 64, 3)


@pytest.mark.parametrize("dtype,chunk,d", [("f32", 16, 64), ("bf16", 64, 32)])
def test_scalar_gate_cuda_core_path(dtype, chunk, d):
    lens = [70, 33, 130]
    inp = synth.draw(sum(lens), 2, d, d, seed=64, dtype=dtype, num_seqs=len(lens), s0_std=0.1)
    inp["cu_seqlens"], inp["num_seqs"] = synth.cu_from_lengths(lens), len(lens)
    _run(inp, chunk, 4)


def test_scalar_gate_long_workload_full_size():
    """B=1, H=16, L=65536: the scalar-gate call equals kda_forward_g given the
    gate broadcast over the channels, bit for bit, at the full size."""
    inp = synth.workload("long")
    d = to_cuda(inp)
    T, H, dk = inp["q"].shape
    gs = synth.scalar_gate(T, H, seed=9).cuda()
    o, S = kda.forward_scalar_gate(d["q"], d["k"], d["v"], gs, d["beta"], num_seqs=1)
    og, Sg = kda.forward_g(d["q"], d["k"], d["v"], gs[:, :, None].expand(T, H, dk).contiguous(),
                           d["beta"], num_seqs=1)
    torch.cuda.synchronize()
    assert torch.equal(o, og) and torch.equal(S, Sg)
