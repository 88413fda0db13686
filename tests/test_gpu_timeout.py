"""The failure path of the bounded device waits (a wait that gives up records
KDA_ERR_TIMEOUT, lets what it issued land, frees its Tensor Memory and
leaves), exercised without any fault: the test hook kda_debug_set_wait_limit
shortens the limit of the first, giving-up waits to a few SM cycles, so the
first wait of each kernel on a copy that cannot have landed yet gives up.
The same workspace then serves a normal call that reports KDA_OK and matches
the float64 oracle."""
import pytest
import torch

from gated_delta_rule_98_b200 import kda, synth
from kda_testutil import assert_close, max_len_of, oracle_forward, to_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H,num_seqs", [(256, 2, 1), (300, 4, 2)])
def test_wait_that_runs_out_reports_timeout_then_recovers(T, H, num_seqs):
    # (256, 2, 1): one sequence cut into segments (preparation, transition and
    # composition, chain pass); (300, 4, 2): two unsegmented sequences
    inp = synth.draw(T, H, 128, 128, seed=60 + T, dtype="bf16", num_seqs=num_seqs, s0_std=0.02)
    inp["num_seqs"] = num_seqs
    d = to_cuda(inp)
    L = max_len_of(inp)
    ws = kda.workspace(num_seqs, T, L, H, 128, 128, torch.bfloat16, 64)
    args = (d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"])
    kw = dict(S0=d["S0"], num_seqs=num_seqs, chunk=64, workspace=ws)
    kda.kda_debug_set_wait_limit(16)
    try:
        kda.forward(*args, **kw)
        torch.cuda.synchronize()
        assert kda.check_device_error(ws) == kda.KDA_ERR_TIMEOUT
    finally:
        kda.kda_debug_set_wait_limit(0)
    o, S = kda.forward(*args, **kw)
    torch.cuda.synchronize()
    assert kda.check_device_error(ws) == kda.KDA_OK
    o_ref, S_ref = oracle_forward(inp)
    assert_close(o, o_ref, torch.bfloat16, "o after recovery")
    assert_close(S, S_ref, torch.bfloat16, "S_final after recovery")
