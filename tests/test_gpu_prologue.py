"""Input prologue (causal depthwise short convolution per sequence, then
Swish): kda_short_conv_swish against the float64 oracle prologue, and
kda_forward_conv (prologue, then the operator) against the oracle prologue
followed by the oracle recurrence, on the segmented and unsegmented
tensor-core paths, packed sequences (empty, shorter than the filter, ragged
tail) and the CUDA-core path."""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, max_len_of, to_cuda

pytestmark = pytest.mark.gpu


def _cu(lens):
    return synth.cu_from_lengths(lens)


@pytest.mark.parametrize("dtype,width,lens", [
    ("bf16", 4, [300, 0, 2, 1, 411, 64]),
    ("f32", 3, [5, 130, 0, 77]),
    ("f32", 1, [40, 24]),
    ("bf16", 2, None),
])
def test_short_conv_swish(dtype, width, lens):
    from oracle import prologue
    H, d = 3, 64
    T = sum(lens) if lens else 4 * 96
    ci = synth.conv_inputs(T, H, d, d, width, seed=71 + width, dtype=dtype)
    x, w = ci["x_q"], ci["w_q"]
    if lens:
        cu = _cu(lens)
        y = kda.short_conv_swish(x.cuda(), w.cuda(), cu_seqlens=cu.cuda(), max_seqlen=max(lens))
        want = prologue.short_conv_swish(x, w, cu_seqlens=cu.numpy())
    else:
        y = kda.short_conv_swish(x.cuda(), w.cuda(), num_seqs=4)
        want = prologue.short_conv_swish(x, w, num_seqs=4)
    torch.cuda.synchronize()
    assert_close(y, want, x.dtype, "prologue")


def _forward_conv(T, H, d, width, dtype, chunk, lens=None, num_seqs=1, seed=0):
    from oracle import prologue, ref
    n_seq = len(lens) if lens else num_seqs
    inp = synth.draw(T, H, d, d, seed=seed, dtype=dtype, num_seqs=n_seq, s0_std=0.02)
    ci = synth.conv_inputs(T, H, d, d, width, seed=seed + 1, dtype=dtype)
    cu = _cu(lens) if lens else None
    inp["cu_seqlens"], inp["num_seqs"] = cu, n_seq
    d_in, d_ci = to_cuda(inp), to_cuda(ci)
    o, S = kda.forward_conv(d_ci["x_q"], d_ci["x_k"], d_ci["x_v"], d_ci["w_q"], d_ci["w_k"],
                            d_ci["w_v"], d_in["z"], d_in["A"], d_in["beta"], S0=d_in["S0"],
                            cu_seqlens=d_in["cu_seqlens"], num_seqs=inp["num_seqs"],
                            max_seqlen=max_len_of(inp), chunk=chunk)
    torch.cuda.synchronize()
    kw = dict(cu_seqlens=None if cu is None else cu.numpy(), num_seqs=inp["num_seqs"])
    q = prologue.short_conv_swish(ci["x_q"], ci["w_q"], **kw)
    k = prologue.short_conv_swish(ci["x_k"], ci["w_k"], **kw)
    v = prologue.short_conv_swish(ci["x_v"], ci["w_v"], **kw)
    o_ref, S_ref = ref.forward(q, k, v, inp["beta"], z=inp["z"], A=inp["A"], S0=inp["S0"],
                               **kw)
    assert_close(o, o_ref, inp["q"].dtype, "o")
    assert_close(S, S_ref, inp["q"].dtype, "S_final")


def test_forward_conv_segmented_tensor_core_path():
    _forward_conv(1024, 4, 128, 4, "bf16", 64, seed=81)


def test_forward_conv_unsegmented_tensor_core_path():
    _forward_conv(8 * 192, 16, 128, 4, "bf16", 64, num_seqs=8, seed=82)


def test_forward_conv_varlen():
    lens = [300, 0, 3, 411, 64]
    _forward_conv(sum(lens), 4, 128, 4, "bf16", 64, lens=lens, seed=83)


@pytest.mark.parametrize("width", [1, 2, 3])
def test_forward_conv_tensor_core_path_short_filters(width):
    # the fused prologue right-aligns taps shorter than 4 (the last on the current token)
    lens = [130, 5, 70]
    _forward_conv(sum(lens), 2, 128, width, "bf16", 64, lens=lens, seed=90 + width)


@pytest.mark.parametrize("dtype,chunk,d,width", [("f32", 16, 64, 4), ("f32", 64, 32, 2),
                                                 ("bf16", 64, 64, 3)])
def test_forward_conv_cuda_core_path(dtype, chunk, d, width):
    lens = [70, 33, 130]
    _forward_conv(sum(lens), 2, d, width, dtype, chunk, lens=lens, seed=84)


def test_forward_conv_long_workload_full_size():
    """B=1, H=16, L=65536 with the prologue fused into the chunk preparation:
    o and S_final against the oracle prologue and recurrence on three sampled
    heads, and, over all heads, agreement with the unfused route (the
    prologue as its own pass, then kda_forward) within the bf16 bar."""
    from oracle import prologue, ref
    from kda_testutil import rel_l2, f64
    inp = synth.workload("long")
    d = to_cuda(inp)
    T, H, dk = inp["q"].shape
    ci_h = synth.conv_inputs(T, H, dk, dk, 4, seed=85)
    ci = to_cuda(ci_h)
    o, S = kda.forward_conv(ci["x_q"], ci["x_k"], ci["x_v"], ci["w_q"], ci["w_k"], ci["w_v"],
                            d["z"], d["A"], d["beta"], num_seqs=1)
    q = kda.short_conv_swish(ci["x_q"], ci["w_q"], num_seqs=1)
    k = kda.short_conv_swish(ci["x_k"], ci["w_k"], num_seqs=1)
    v = kda.short_conv_swish(ci["x_v"], ci["w_v"], num_seqs=1)
    o2, S2 = kda.forward(q, k, v, d["z"], d["A"], d["beta"], num_seqs=1)
    torch.cuda.synchronize()
    assert rel_l2(f64(o), f64(o2)) <= 5e-3 and rel_l2(f64(S), f64(S2)) <= 5e-3
    heads = [0, 7, 15]
    rows = lambda w, d_: w.reshape(H, d_, -1)[heads].reshape(len(heads) * d_, -1)
    xs = {key: ci_h[key][:, heads] for key in ("x_q", "x_k", "x_v")}
    qh = prologue.short_conv_swish(xs["x_q"], rows(ci_h["w_q"], dk))
    kh = prologue.short_conv_swish(xs["x_k"], rows(ci_h["w_k"], dk))
    vh = prologue.short_conv_swish(xs["x_v"], rows(ci_h["w_v"], dk))
    o_ref, S_ref = ref.forward(qh, kh, vh, inp["beta"][:, heads], z=inp["z"][:, heads],
                               A=inp["A"][heads], num_seqs=1)
    assert_close(o[:, heads], o_ref, torch.bfloat16, "o, sampled heads")
    assert_close(S[:, heads], S_ref, torch.bfloat16, "S_final, sampled heads")
