"""The multi-rank logic of bench.py on CPU: two gloo ranks, no GPU.

bench.py --gpus N runs one independent problem per rank (weak scaling) and
reports the max over ranks of the device time; these tests exercise that
aggregation and the reference arm's rank-0-only behaviour with world size 2.
"""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = bench.max_over_ranks(ms_local, world)
    value = bench.weak_scaling_value(1000, world, ms)
    out.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_value_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 15.0                          # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 1000 / 0.015)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(64, 1, 2.0) == pytest.approx(32000.0)


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.parametrize("steps", [1])
def test_reference_arm_json_line(steps):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", str(steps), "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _cp_worker(rank, world, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import bench
    from gated_delta_rule_98_b200 import cp
    from oracle import ref
    from test_cp_host import _OracleOps, _problem
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    T = 150
    p = _problem(3, T, 2, 6, 4, s0=0.0)
    a, b = bench.shard_bounds(T, world, rank)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    o_sh, S_after = cp.context_parallel_forward(t(p["q"][a:b]), t(p["k"][a:b]), t(p["v"][a:b]),
                                                t(p["z"][a:b]), t(p["A"]), t(p["beta"][a:b]),
                                                max_seqlen=b - a, ops=_OracleOps())
    o_ref, S_ref = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], num_seqs=1)
    err, rel, serr = bench.cp_parity(o_sh, t(o_ref[a:b]), S_after[0], t(S_ref[0]),
                                     rank == world - 1, world)
    ms = bench.max_over_ranks(4.0 + rank, world)
    out.put((rank, a, b, err, rel, serr, ms, bench.strong_scaling_value(T, ms)))
    dist.barrier()
    dist.destroy_process_group()


def test_context_parallel_mode_aggregation_with_gloo():
    """bench.py --mode cp on CPU ranks: the shards tile the sequence in chunk
    multiples, the parity reduction sees the sharded result equal to the
    one-pass oracle on every rank, and the strong-scaling throughput divides
    the whole sequence by the slowest rank's time."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + os.getpid() % 1000
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == 0 and res[0][2] == res[1][1] and res[1][2] == 150
    assert res[0][2] % 64 == 0
    for rank, a, b, err, rel, serr, ms, value in res:
        assert err < 1e-10 and rel < 1e-10 and serr < 1e-10
        assert ms == 5.0 and value == pytest.approx(150 / 0.005)
