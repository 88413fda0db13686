"""kda_forward_noalloc compared with kda_forward.

kda_forward_noalloc is for callers that cannot allocate device memory: a host
whose GPU memory belongs to another allocator (so a new cudaMalloc fails or
fragments that pool), or code that must not call cudaMalloc/cudaFree because
they can synchronise the whole device.  It runs the same operator on a fixed
scratch array that the library defines, so the caller passes only inputs and
outputs.  Here it is called through the C ABI twice in a row, on two
different problems, and each result is compared with kda_forward run on a
caller-allocated workspace, within the tolerances of the other GPU tests.
This file sorts last so that a run stopping at its first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, f64, gpu_forward, max_len_of, to_cuda

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(inp, chunk):
    d = to_cuda(inp)
    T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    N = inp["num_seqs"]
    o = torch.full((T, H, dv), float("nan"), dtype=d["q"].dtype, device="cuda")
    S = torch.full((N, H, dk, dv), float("nan"), device="cuda")
    dt = kda.KDA_BF16 if d["q"].dtype == torch.bfloat16 else kda.KDA_F32
    st = kda.kda_forward_noalloc(
        _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["z"]), _p(d["A"]), _p(d["beta"]),
        _p(d.get("S0")), _p(d.get("cu_seqlens")), N, T, max_len_of(inp), H, dk, dv, dt, chunk,
        _p(o), _p(S), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kda.KDA_OK, kda.status_string(st)
    torch.cuda.synchronize()
    return o, S


def _cases():
    lens = [300, 5, 0, 411]
    a = synth.draw(sum(lens), 4, 128, 128, seed=31, dtype="bf16", num_seqs=len(lens),
                   s0_std=0.02)
    a["cu_seqlens"] = synth.cu_from_lengths(lens)
    a["num_seqs"] = len(lens)
    b = synth.draw(2 * 333, 3, 64, 32, seed=32, dtype="f32", num_seqs=2, s0_std=None)
    b["cu_seqlens"] = None
    b["num_seqs"] = 2
    return [(a, 64, torch.bfloat16), (b, 16, torch.float32)]


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    cases = _cases()
    results = [_noalloc(inp, chunk) for inp, chunk, _ in cases]   # two calls back to back
    for (inp, chunk, dt), (o_na, S_na) in zip(cases, results):
        o_ref, S_ref = gpu_forward(inp, chunk=chunk)
        assert_close(o_na, f64(o_ref), dt, "o")
        assert_close(S_na, f64(S_ref), dt, "S_final")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # fp32 inputs take the CUDA-core path, whose scratch grows with the tokens
    T, H, D = 1 << 16, 16, 128
    need = kda.kda_forward_workspace_size(1, T, T, H, D, D, kda.KDA_F32, 64)
    assert need > kda.KDA_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    st = kda.kda_forward_noalloc(fake, fake, fake, fake, fake, fake, None, None, 1, T, T, H, D, D,
                                 kda.KDA_F32, 64, fake, fake, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
