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
