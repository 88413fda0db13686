"""Context parallelism on CPU: the float64 sharded computation pinned to the
unsharded oracle, and the collective logic of ``cp.context_parallel_forward``
with two gloo ranks driving oracle-based per-rank steps (no GPU)."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import cp as ocp
from oracle import ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _problem(seed, T, H, dk, dv, s0=0.3, z_shift=-6.0):
    """z is shifted down so that the decay is weak (alpha near 1) and the shard
    maps M stay far from zero: the fold order then matters."""
    rng = np.random.default_rng(seed)
    return dict(q=rng.standard_normal((T, H, dk)), k=rng.standard_normal((T, H, dk)),
                v=rng.standard_normal((T, H, dv)),
                beta=1 / (1 + np.exp(-rng.standard_normal((T, H)))),
                z=rng.standard_normal((T, H, dk)) + z_shift, A=rng.standard_normal(H),
                S0=rng.standard_normal((1, H, dk, dv)) * s0)


def _cut(p, a, b):
    return {key: (val[a:b] if key in ("q", "k", "v", "beta", "z") else val)
            for key, val in p.items()}


def test_transition_product_equals_zero_value_run_from_identity():
    """M of a shard (product of transitions) is the state a run with v = 0
    leaves from S0 = I: the recurrence is linear in the state."""
    p = _problem(1, 11, 2, 5, 5)
    M, N = ocp.shard_transition(p["q"], p["k"], p["v"], p["beta"], p["z"], p["A"])
    eye = np.broadcast_to(np.eye(5), (1, 2, 5, 5)).copy()
    _, S = ref.forward(p["q"], p["k"], np.zeros_like(p["v"]), p["beta"], z=p["z"], A=p["A"],
                       S0=eye, num_seqs=1)
    assert np.abs(S[0] - M).max() < 1e-12
    _, S0run = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], num_seqs=1)
    assert np.abs(S0run[0] - N).max() < 1e-12


@pytest.mark.parametrize("cuts", [[0, 7, 19, 30], [0, 1, 2, 30], [0, 15, 15, 30]])
def test_sharded_oracle_equals_one_pass(cuts):
    p = _problem(2, 30, 2, 6, 4)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                        num_seqs=1)
    Ms, Ns = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        s = _cut(p, a, b)
        M, N = ocp.shard_transition(s["q"], s["k"], s["v"], s["beta"], s["z"], s["A"])
        Ms.append(M)
        Ns.append(N)
    S_ins = ocp.prefix_states(Ms, Ns, p["S0"][0])
    outs = []
    for r, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        s = _cut(p, a, b)
        o_r, S_r = ref.forward(s["q"], s["k"], s["v"], s["beta"], z=s["z"], A=s["A"],
                               S0=S_ins[r][None], num_seqs=1)
        outs.append(o_r)
    assert np.abs(np.concatenate(outs) - o).max() < 1e-12
    assert np.abs(S_r - Sf).max() < 1e-12
    # the maps matter here: folding them in the wrong order changes the result
    if len(Ms) > 2 and all(b > a for a, b in zip(cuts[:-1], cuts[1:])):
        wrong = ocp.prefix_states(Ms[::-1], Ns[::-1], p["S0"][0])[-1]
        assert np.abs(wrong - S_ins[-1]).max() > 1e-3


class _OracleOps:
    """Per-rank steps in float64 on CPU, standing in for the GPU kernels."""

    def local(self, q, k, v, z, A, beta, cu_seqlens, max_seqlen, chunk):
        M, N = ocp.shard_transition(q, k, v, beta, z, A)
        shard = (q, k, v, z, A, beta)
        return torch.from_numpy(M)[None], torch.from_numpy(N)[None], shard

    def compose(self, M, N, S):
        return torch.from_numpy(ocp.compose(M[0].numpy(), N[0].numpy(),
                                            None if S is None else S[0].numpy()))[None]

    def finish(self, shard, S_in):
        q, k, v, z, A, beta = shard
        o, S = ref.forward(q, k, v, beta, z=z, A=A,
                           S0=None if S_in is None else S_in.numpy(), num_seqs=1)
        return torch.from_numpy(o), torch.from_numpy(S)


def _worker(rank, world, port, cuts, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from gated_delta_rule_98_b200 import cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    p = _problem(3, cuts[-1], 2, 6, 4)
    s = {key: torch.from_numpy(np.ascontiguousarray(val)) for key, val in
         _cut(p, cuts[rank], cuts[rank + 1]).items()}
    o, S = cp.context_parallel_forward(s["q"], s["k"], s["v"], s["z"], s["A"], s["beta"],
                                       S0=s["S0"], ops=_OracleOps())
    out.put((rank, o.numpy(), S.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 13, 29], [0, 1, 12, 20]])
def test_context_parallel_forward_gloo_ranks(cuts):
    """Two ranks, then three (one holding a single token): rank r folds the
    maps of ranks 0 .. r-1 in order."""
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + os.getpid() % 1000 + 7 * world
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = _problem(3, cuts[-1], 2, 6, 4)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                        num_seqs=1)
    assert np.abs(np.concatenate([r[1] for r in res]) - o).max() < 1e-12
    assert np.abs(res[-1][2] - Sf).max() < 1e-12
