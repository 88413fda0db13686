"""GPU parity of kda_forward / kda_forward_g against the float64 oracle.

Inputs come from the seeded generators; the oracle sees the same rounded
values.  Sizes span several chunks and ragged tails; the full-length
workload is checked on every head and token.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, f64, gpu_forward, oracle_forward, to_cuda

pytestmark = pytest.mark.gpu


def test_tiny_fp32_workload():
    inp = synth.workload("tiny")
    o, S = gpu_forward(inp, chunk=16)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(S, S_ref, torch.float32, "S_final")


def test_bf16_L4096_workload():
    inp = synth.workload("bf16")
    o, S = gpu_forward(inp, chunk=64)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S_final")


def test_varlen_workload():
    inp = synth.workload("varlen")
    o, S = gpu_forward(inp, chunk=64)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S_final")


def test_long_workload_all_heads():
    """The bench's workload (B=1, H=16, L=65536) in full: every head and token."""
    inp = synth.workload("long")
    o, S = gpu_forward(inp, chunk=64)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S_final")


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 32)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_shapes_ragged_varlen(dk, dv, dtype):
    lens = [1, 77, 0, 130, 16, 64, 63]
    T = sum(lens)
    inp = synth.draw(T, 3, dk, dv, seed=100 + dk + dv, dtype=dtype, num_seqs=len(lens),
                     s0_std=0.3)
    inp["cu_seqlens"] = synth.cu_from_lengths(lens)
    inp["num_seqs"] = len(lens)
    o_ref, S_ref = oracle_forward(inp)
    for chunk in (16, 64):
        o, S = gpu_forward(inp, chunk=chunk)
        dt = torch.float32 if dtype == "f32" else torch.bfloat16
        assert_close(o, o_ref, dt, f"o chunk={chunk}")
        assert_close(S, S_ref, dt, f"S_final chunk={chunk}")


def test_chunk16_equals_chunk64():
    inp = synth.draw(700, 4, 128, 128, seed=7, dtype="bf16", s0_std=0.02)
    o16, S16 = gpu_forward(inp, chunk=16)
    o64, S64 = gpu_forward(inp, chunk=64)
    assert_close(o16, f64(o64), torch.bfloat16, "o")
    assert_close(S16, f64(S64), torch.bfloat16, "S")


def test_packed_equals_separate_calls():
    lens = [200, 333, 91]
    inp = synth.draw(sum(lens), 4, 64, 64, seed=8, dtype="bf16", num_seqs=3, s0_std=0.1)
    inp["cu_seqlens"] = synth.cu_from_lengths(lens)
    inp["num_seqs"] = 3
    o, S = gpu_forward(inp)
    a = 0
    for n, L in enumerate(lens):
        part = {key: inp[key][a:a + L] for key in ("q", "k", "v", "z", "beta")}
        part.update(A=inp["A"], S0=inp["S0"][n:n + 1], cu_seqlens=None, num_seqs=1)
        o1, S1 = gpu_forward(part)
        assert torch.equal(o1, o[a:a + L]) or np.abs(f64(o1) - f64(o[a:a + L])).max() < 1e-6
        assert np.abs(f64(S1[0]) - f64(S[n])).max() < 1e-5
        a += L


def test_state_passing_split_equals_one_call():
    inp = synth.draw(1000, 2, 128, 128, seed=9, dtype="bf16", s0_std=0.02)
    o, S = gpu_forward(inp)
    cut = 421
    first = {key: inp[key][:cut] for key in ("q", "k", "v", "z", "beta")}
    first.update(A=inp["A"], S0=inp["S0"], num_seqs=1)
    second = {key: inp[key][cut:] for key in ("q", "k", "v", "z", "beta")}
    second.update(A=inp["A"], num_seqs=1)
    o1, S1 = gpu_forward(first)
    o2, S2 = gpu_forward(second, S0=S1)
    assert_close(torch.cat([o1, o2]), f64(o), torch.bfloat16, "o")
    assert_close(S2, f64(S), torch.bfloat16, "S")


def test_in_place_state_passing():
    inp = synth.draw(300, 2, 64, 64, seed=10, dtype="f32", s0_std=0.2)
    o_ref, S_ref = oracle_forward(inp)
    d = to_cuda(inp)
    S = d["S0"].clone()
    o, _ = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], S0=S, S_final=S,
                       num_seqs=1, chunk=64)
    torch.cuda.synchronize()
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(S, S_ref, torch.float32, "S in place")


def test_prefill_equals_repeated_decode():
    T, H = 37, 3
    inp = synth.draw(T, H, 128, 128, seed=11, dtype="bf16", s0_std=0.02)
    o, S = gpu_forward(inp)
    d = to_cuda(inp)
    St = d["S0"].clone()
    outs = []
    for t in range(T):
        tok = {key: d[key][t:t + 1].clone() for key in ("q", "k", "v", "z", "beta")}
        outs.append(kda.decode_step(tok["q"], tok["k"], tok["v"], tok["z"], d["A"], tok["beta"],
                                    St))
    torch.cuda.synchronize()
    assert_close(torch.cat(outs), f64(o), torch.bfloat16, "o")
    assert_close(St, f64(S), torch.bfloat16, "S")


# ------------------------------------------------- g-entry special cases ---

def test_g_entry_deltanet_and_scalar_gate():
    """alpha = 1 (g = 0) is DeltaNet; one g per head is Gated DeltaNet."""
    rng = np.random.default_rng(12)
    T, H = 200, 2
    inp = synth.draw(T, H, 64, 64, seed=12, dtype="f32", s0_std=0.1)
    g0 = torch.zeros(T, H, 64)
    o, S = gpu_forward(inp, g=g0)
    o_ref, S_ref = oracle_forward(inp, g=g0)
    assert_close(o, o_ref, torch.float32, "DeltaNet o")
    assert_close(S, S_ref, torch.float32, "DeltaNet S")
    gs = torch.from_numpy(-5.0 * rng.random((T, H, 1))).float().expand(T, H, 64).contiguous()
    o, S = gpu_forward(inp, g=gs)
    o_ref, S_ref = oracle_forward(inp, g=gs)
    assert_close(o, o_ref, torch.float32, "GDN o")
    assert_close(S, S_ref, torch.float32, "GDN S")


def test_strongest_decay_everywhere():
    """g = -5 on every channel: the chunk-local log-decay reaches -320."""
    inp = synth.draw(256, 2, 128, 128, seed=13, dtype="bf16", s0_std=0.02)
    g = torch.full((256, 2, 128), -5.0)
    o, S = gpu_forward(inp, g=g)
    o_ref, S_ref = oracle_forward(inp, g=g)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


def test_weak_decay_long_memory_segmented():
    """z shifted down so most channels barely decay (alpha^4096 mostly above
    1e-3): the segment transitions M_p stay far from zero and every segment's
    incoming state depends on them.  H = 4, L = 4096: 16 segments per head."""
    inp = synth.draw(4096, 4, 128, 128, seed=131, dtype="bf16", num_seqs=1, s0_std=0.02)
    inp["z"] = (inp["z"].float() - 8.0).to(torch.bfloat16)
    inp["cu_seqlens"], inp["num_seqs"] = None, 1
    o, S = gpu_forward(inp)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S_final")


def test_beta_zero_gives_pure_decay():
    inp = synth.draw(130, 2, 64, 64, seed=14, dtype="f32", s0_std=0.5)
    inp["beta"] = torch.zeros_like(inp["beta"])
    o, S = gpu_forward(inp)
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(S, S_ref, torch.float32, "S")


# ------------------------------------------------------ device-side errors ---

@pytest.mark.parametrize("cu", [[0, 10, 5, 40], [0, 10, 20, 39], [1, 10, 20, 40],
                                [0, 30, 35, 40]])
def test_bad_cu_seqlens_reported_and_nothing_written(cu):
    inp = synth.draw(40, 2, 32, 32, seed=15, dtype="f32", num_seqs=3, s0_std=0.1)
    d = to_cuda(inp)
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    ws = kda.workspace(3, 40, 20, 2, 32, 32, torch.float32, 16)
    o = torch.full((40, 2, 32), 7.0, device="cuda")
    Sf = torch.full((3, 2, 32, 32), 7.0, device="cuda")
    kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], S0=d["S0"], cu_seqlens=cu_t,
                max_seqlen=20, chunk=16, o=o, S_final=Sf, workspace=ws)
    assert kda.check_device_error(ws) == kda.KDA_ERR_INVALID_ARG
    assert bool((o == 7.0).all()) and bool((Sf == 7.0).all())
    # the same workspace then serves a valid call and reports OK
    good = torch.tensor([0, 10, 25, 40], dtype=torch.int32, device="cuda")
    kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], S0=d["S0"], cu_seqlens=good,
                max_seqlen=20, chunk=16, o=o, S_final=Sf, workspace=ws)
    assert kda.check_device_error(ws) == kda.KDA_OK


def test_all_sequences_empty():
    inp = synth.draw(0, 2, 32, 32, seed=16, dtype="f32", num_seqs=2, s0_std=0.1)
    inp["cu_seqlens"] = torch.zeros(3, dtype=torch.int32)
    inp["num_seqs"] = 2
    o, S = gpu_forward(inp)
    assert o.numel() == 0
    assert torch.equal(S.cpu(), inp["S0"])
