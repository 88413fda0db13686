"""GPU parity of kda_decode_step against the float64 oracle."""
import numpy as np
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, f64

pytestmark = pytest.mark.gpu


def test_decode_workload_1000_steps_sampled():
    """B=256, H=16, d=128: all states advance on the GPU for 1000 steps; a
    fixed sample of (sequence, head) pairs is followed by the oracle, and o and
    S are compared after 1, 10, 100 and 1000 steps."""
    from oracle import ref
    B, H, D = 256, 16, 128
    A, S0 = synth.decode_state(B, H, D, D)
    S = S0.cuda()
    Ad = A.cuda()
    rng = np.random.default_rng(99)
    bs = np.sort(rng.choice(B, 48, replace=False))
    hs = rng.integers(0, H, 48)
    pick = lambda t: f64(t)[bs, hs][:, None]     # 48 sampled pairs as 48 one-head sequences
    S_ref = f64(S0)[bs, hs][:, None]
    for step in range(1000):
        tok = synth.decode_token(step, B, H, D, D)
        d = {key: t.cuda() for key, t in tok.items()}
        o = kda.decode_step(d["q"], d["k"], d["v"], d["z"], Ad, d["beta"], S)
        g = ref.gate(f64(tok["z"]), f64(A))[bs, hs][:, None]   # each pair keeps its head's A
        o_ref, S_ref = ref.decode_step(pick(tok["q"]), pick(tok["k"]), pick(tok["v"]),
                                       f64(tok["beta"])[bs, hs][:, None], S_ref, g=g)
        if step + 1 in (1, 10, 100, 1000):
            torch.cuda.synchronize()
            assert_close(o[bs, hs], o_ref[:, 0], torch.bfloat16, f"o step {step + 1}")
            assert_close(S[bs, hs], S_ref[:, 0], torch.bfloat16, f"S step {step + 1}")


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_shapes(dk, dv, dtype):
    from oracle import ref
    B, H = 5, 3
    inp = synth.draw(B, H, dk, dv, seed=dk * 3 + dv, dtype=dtype, num_seqs=B, s0_std=0.2)
    S = inp["S0"].cuda()
    o = kda.decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["z"].cuda(),
                        inp["A"].cuda(), inp["beta"].cuda(), S)
    torch.cuda.synchronize()
    o_ref, S_ref = ref.decode_step(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"],
                                   z=inp["z"], A=inp["A"])
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    assert_close(o, o_ref, dt, "o")
    assert_close(S, S_ref, dt, "S")


@pytest.mark.parametrize("dtype,width,dk,dv,steps", [("bf16", 4, 128, 128, 120),
                                                     ("f32", 2, 64, 32, 100),
                                                     ("bf16", 1, 32, 64, 100)])
def test_decode_conv_rolling_window(dtype, width, dk, dv, steps):
    """kda_decode_step_conv for `steps` tokens of B sequences, the window
    starting at zeros, against the oracle prologue over each whole sequence
    followed by the oracle decode step token by token: every step's o, the
    final state, and the window after the last step (the last width - 1 raw
    inputs, exactly)."""
    from oracle import prologue, ref
    B, H = 3, 2
    T = B * steps                                # sequence b: tokens b*steps .. (b+1)*steps - 1
    ci = synth.conv_inputs(T, H, dk, dv, width, seed=140 + width, dtype=dtype)
    inp = synth.draw(T, H, dk, dv, seed=141 + width, dtype=dtype, num_seqs=B, s0_std=0.05)
    q = prologue.short_conv_swish(ci["x_q"], ci["w_q"], num_seqs=B)
    k = prologue.short_conv_swish(ci["x_k"], ci["w_k"], num_seqs=B)
    v = prologue.short_conv_swish(ci["x_v"], ci["w_v"], num_seqs=B)
    at = lambda x, t: x.reshape(B, steps, *x.shape[1:])[:, t]   # token t of every sequence
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    w = {key: ci[key].cuda() for key in ("w_q", "w_k", "w_v")}
    state = kda.conv_state_zeros(B, H, dk, dv, width, dt)
    S = inp["S0"].cuda()
    A = inp["A"].cuda()
    S_ref = f64(inp["S0"])
    outs, refs = [], []
    for t in range(steps):
        o = kda.decode_step_conv(at(ci["x_q"], t).cuda(), at(ci["x_k"], t).cuda(),
                                 at(ci["x_v"], t).cuda(), w["w_q"], w["w_k"], w["w_v"], state,
                                 at(inp["z"], t).cuda(), A, at(inp["beta"], t).cuda(), S)
        outs.append(o)
        o_ref, S_ref = ref.decode_step(at(q, t), at(k, t), at(v, t), f64(at(inp["beta"], t)),
                                       S_ref, z=f64(at(inp["z"], t)), A=f64(inp["A"]))
        refs.append(o_ref)
    torch.cuda.synchronize()
    assert_close(torch.stack(outs, 1), np.stack(refs, 1), dt, "o, every step")
    assert_close(S, S_ref, dt, "S after the last step")
    if width > 1:
        last = lambda x: x.reshape(B, steps, H * x.shape[-1])[:, steps - width + 1:]
        want = torch.cat([last(ci["x_q"]), last(ci["x_k"]), last(ci["x_v"])], 2)  # [B, W-1, C]
        assert torch.equal(state.cpu(), want.transpose(1, 2).contiguous())
