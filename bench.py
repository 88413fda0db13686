#!/usr/bin/env python
"""KDA operator benchmark: prefill tokens/s on B=1, H=16, d=128, L=65536 (bf16
inputs, fp32 state, chunk 64) plus decode steps/s on B=256, H=16, d=128.

One JSON line on rank 0.  A step is one kda_forward over the whole prefill
workload (gate, normalisation, chunk cumsum, intra-chunk products, UT
inverse, WY blocks, state pass, final state).  The decode step (the remaining
hot-path row) is measured in the same run and reported under "decode".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own copy of the
workload (independent problems, no data-path collective: weak scaling); the
time is the max over ranks.  ``--impl reference`` times the float64 CPU oracle
on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, H, D, L_DEFAULT, CHUNK = 1, 16, 128, 65536, 64
DEC_B = 256
METRIC = "KDA prefill tokens/s (B=1,H=16,d=128,L=64k) & decode steps/s; % tensor/HBM roofline"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def alg_flops(T, C=CHUNK, d=D, heads=H):
    """Kimi Linear summary §6.3: 6 T d^2 + 3 T C d + T C^2 per head."""
    return heads * (6 * T * d * d + 3 * T * C * d + T * C * C)


def alg_bytes_prefill(T, N=1, heads=H, dk=D, dv=D, elt=2, s0=False, sfinal=True):
    """q, k, z, v, beta read and o written per token-head, plus states."""
    per_tok = elt * (3 * dk + dv + 1 + dv)
    st = N * heads * dk * dv * 4
    return T * heads * per_tok + (st if s0 else 0) + (st if sfinal else 0)


def alg_bytes_decode(Bd=DEC_B, heads=H, dk=D, dv=D, elt=2):
    """State read + written, q, k, z, v, beta read and o written per (b, h)."""
    return Bd * heads * (2 * dk * dv * 4 + elt * (3 * dk + dv + 1 + dv))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, src="fallback")


# The sources each recorded kernel's traffic depends on (a change elsewhere
# leaves its record valid).
_TRAFFIC_SOURCES = {
    "forward": ("kda_prep_tc.cu", "kda_prefill_tc.cu", "kda_tc_common.cuh", "tc_sm100.cuh",
                "kda_common.cuh", "kda_launch.h"),
    "decode": ("kda_decode.cu", "kda_common.cuh", "kda_launch.h"),
}


def kernel_source_hash(kind):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_98_b200", "csrc")
    for fn in sorted(_TRAFFIC_SOURCES[kind]):
        h.update(fn.encode())
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kind):
    """ncu DRAM bytes per launch recorded for the current kernel sources, or None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kind)
    if not e or e.get("source_hash") != kernel_source_hash(kind):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 10 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.f = None
        self.start = 0

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        # nvidia-smi takes a while to start: wait (at most 5 s) for its first
        # sample so that the timed region is covered from its start
        t_end = time.time() + 5.0
        while time.time() < t_end and os.path.getsize(self.f.name) == 0:
            time.sleep(0.01)
        return self

    def mark(self):
        """Only samples written after this call count (call it when the timed region starts)."""
        if self.proc is not None:
            self.start = os.path.getsize(self.f.name)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return None
        self.f.flush()
        with open(self.f.name) as fh:
            fh.seek(self.start)
            rows = [r.split(",") for r in fh.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for nm, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x, world, device=None):
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, ms_max):
    """Whole-job throughput: every rank processed units_per_rank in ms_max."""
    return world * units_per_rank / (ms_max / 1e3)


def time_configs(dev, stream, pk, world, rank_max, barrier, warmup, log_fn):
    """ms per kda_forward call, tokens/s and HBM roofline fraction of the other
    prefill configurations: the bf16 L=4096 workload, the long workload's
    length sweep and the packed varlen workload (H=32, nonzero S0)."""
    import torch

    from gated_delta_rule_98_b200 import kda, synth
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    res = {}
    for name, wl, L in (("bf16_L4096", "bf16", None), ("long_L2048", "long", 2048),
                        ("long_L8192", "long", 8192), ("long_L32768", "long", 32768),
                        ("varlen_T32768_H32", "varlen", None)):
        inp = synth.workload(wl, L=L)
        T, Hh = inp["q"].shape[0], inp["q"].shape[1]
        N = inp["num_seqs"]
        cu = inp.get("cu_seqlens")
        max_len = int((cu[1:] - cu[:-1]).max()) if cu is not None else T // N
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        o = torch.empty((T, Hh, D), dtype=torch.bfloat16, device=dev)
        Sf = torch.empty((N, Hh, D, D), dtype=torch.float32, device=dev)
        ws = kda.workspace(N, T, max_len, Hh, D, D, torch.bfloat16, CHUNK, device=dev)

        def fwd():
            kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], S0=d.get("S0"),
                        cu_seqlens=d.get("cu_seqlens"), num_seqs=N, max_seqlen=max_len,
                        chunk=CHUNK, o=o, S_final=Sf, workspace=ws, stream=stream)

        for _ in range(warmup):
            fwd()
        torch.cuda.synchronize()
        assert kda.check_device_error(ws) == kda.KDA_OK
        # enough calls for about 0.1 s of device time
        e0.record(stream)
        fwd()
        e1.record(stream)
        torch.cuda.synchronize()
        n = int(min(2000, max(20, 100.0 / max(e0.elapsed_time(e1), 1e-3))))
        barrier()
        e0.record(stream)
        for _ in range(n):
            fwd()
        e1.record(stream)
        torch.cuda.synchronize()
        ms_local = e0.elapsed_time(e1) / n
        ms = rank_max(ms_local)
        nbytes = alg_bytes_prefill(T, N=N, heads=Hh, s0=cu is not None)
        flops = alg_flops(T, heads=Hh)
        ach = nbytes / (ms_local / 1e3) / 1e9
        res[name] = {"ms_per_call": ms, "calls": n, "tokens_per_s": world * T / (ms / 1e3),
                     "B_or_N": N, "H": Hh, "tokens": T, "alg_bytes": nbytes,
                     "achieved_gbs": ach, "hbm_frac": ach / pk["hbm"],
                     "roofline_time_us": max(nbytes / pk["hbm"] / 1e3, flops / pk["bf16"] / 1e6),
                     "tensor_flops_frac": flops / (ms_local / 1e3) / 1e12 / pk["bf16"],
                     "launches": kda.kda_forward_launches(N, T, max_len, Hh, D, D, kda.KDA_BF16,
                                                          CHUNK)}
        log_fn(f"config {name}: {ms:.4f} ms/call, {res[name]['hbm_frac']:.3f} of HBM")
        del d, o, Sf, ws
        torch.cuda.empty_cache()
    return res


def strong_scaling_value(total_units, ms_max):
    """Whole-job throughput when the ranks share one problem of total_units."""
    return total_units / (ms_max / 1e3)


def shard_bounds(T, world, rank):
    """Contiguous token range [a, b) of rank `rank` out of `world` (chunk-aligned)."""
    per = ((T + world - 1) // world + CHUNK - 1) // CHUNK * CHUNK
    a = min(T, rank * per)
    return a, min(T, a + per)


def cp_parity(o_shard, o_ref_shard, S_after, S_ref, last, world, device=None):
    """Agreement of a context-parallel run with the single-GPU call, reduced over
    the ranks: (max-abs over sampled o rows, their relative L2, max-abs of the
    final state held by the last rank)."""
    import torch
    rows = torch.arange(0, o_shard.shape[0], 97, device=o_shard.device)
    g, w = o_shard[rows].double(), o_ref_shard[rows].double()
    err = float((g - w).abs().max()) if rows.numel() else 0.0
    num, den = float(((g - w) ** 2).sum()), float((w ** 2).sum())
    serr = float((S_after.double() - S_ref.double()).abs().max()) if last else 0.0
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([err, serr], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        n = torch.tensor([num, den], dtype=torch.float64, device=device)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
        err, serr, num, den = float(t[0]), float(t[1]), float(n[0]), float(n[1])
    return err, (num / den) ** 0.5 if den > 0 else 0.0, serr


def run_cp(args):
    """Context parallelism: one sequence of args.L tokens split into contiguous
    shards, one per rank (strong scaling); a step is one
    cp.context_parallel_forward (local pass, one all-gather of the shard maps,
    prefix fold, finishing pass)."""
    import datetime

    import torch
    import torch.distributed as dist

    from gated_delta_rule_98_b200 import cp, kda, synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    L = args.L
    inp = synth.workload("long", L=L)
    d = {k_: (v_.to(dev) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    a, b = shard_bounds(L, world, rank)
    sh = {k_: d[k_][a:b].contiguous() for k_ in ("q", "k", "v", "z", "beta")}
    # the single-GPU call on the whole sequence (untimed), for the parity check
    o_ref, S_ref = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], num_seqs=1,
                               chunk=CHUNK)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step(ev=None):
        return cp.context_parallel_forward(sh["q"], sh["k"], sh["v"], sh["z"], d["A"], sh["beta"],
                                           max_seqlen=b - a, chunk=CHUNK, events=ev)

    for _ in range(args.warmup):
        o_sh, S_after = step()
    torch.cuda.synchronize()
    err, rel, serr = cp_parity(o_sh, o_ref[a:b], S_after[0], S_ref[0], rank == world - 1, world,
                               dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ag_ms = 0.0
    e0.record(stream)
    for _ in range(args.steps):
        step((g0, g1))
        g1.synchronize()
        ag_ms += g0.elapsed_time(g1)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, world, dev)
    ag = max_over_ranks(ag_ms / args.steps, world, dev)
    fl = kda.kda_forward_launches(1, b - a, b - a, H, D, D, kda.KDA_BF16, CHUNK)
    launches = 3 + rank + (2 if fl == 4 else 1)  # local pass, folds, finishing pass
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": strong_scaling_value(L, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "mode": "context_parallel",
        "config": {"workload": f"KDA fwd long, one sequence split over the ranks: B=1 H={H} "
                               f"L={L} dk=dv={D}, bf16 inputs, fp32 state, chunk {CHUNK}",
                   "B": 1, "H": H, "L": L, "shard_tokens": b - a,
                   "parallelism": f"context parallel x{world} (one all-gather of the shard maps)"},
        "allgather_ms": ag, "allgather_share": ag / ms if ms > 0 else None,
        "parity_vs_single_gpu": {"o_sampled_max_abs": err, "o_sampled_rel_l2": rel,
                                 "S_final_max_abs": serr, "bar": "max-abs 2e-2, rel-L2 5e-3"},
        "gpu_launches": launches * args.steps,
    }), flush=True)


def oracle_baseline(inp, n_tokens):
    """Float64 oracle on the first n_tokens of the workload (all heads)."""
    from oracle import ref
    sl = slice(0, n_tokens)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    ref.forward(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["beta"][sl], z=inp["z"][sl],
                A=inp["A"], num_seqs=1, threads=threads)
    dt = time.perf_counter() - t0
    return dt, min(threads, H)


def run_reference(args):
    """The reference arm: the float64 CPU oracle, timed on a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from gated_delta_rule_98_b200 import synth
    n_tok = 4096
    inp = synth.draw(n_tok, H, D, D, seed=2, dtype="bf16")  # same generators, shorter draw
    times = []
    for i in range(args.warmup + args.steps):
        dt, cores = oracle_baseline(inp, n_tok)
        if i >= args.warmup:
            times.append(dt)
    t = sum(times) / len(times)
    val = n_tok / t
    sample = f"{n_tok} tokens x {H} heads (B=1, d=128, bf16-rounded inputs widened to f64)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "KDA fwd long (float64 CPU oracle, bounded sample)", "B": 1,
                   "H": H, "L": L_DEFAULT, "dk": D, "dv": D, "sample_tokens": n_tok},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=360)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--mode", choices=["weak", "cp"], default="weak",
                    help="weak: one independent problem per rank (default); cp: one sequence "
                         "split over the ranks (context parallelism, strong scaling)")
    ap.add_argument("--L", type=int, default=L_DEFAULT, help="prefill length (sweep)")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other prefill configurations (profiling captures)")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run one part (profiling captures); the other part is reported as null")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.mode == "cp":
        return run_cp(args)

    import torch
    import torch.distributed as dist

    from gated_delta_rule_98_b200 import kda, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x):
        return max_over_ranks(x, world, dev)

    L = args.L
    T = B * L
    log(f"[rank {rank}] generating inputs L={L}")
    inp = synth.workload("long", L=L)
    stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    pk = peaks()
    out = {"ms": None, "value": None, "roofline": None, "e2e": None, "clocks": None,
           "launches": 0, "decode": None, "variants": None, "configs": None}

    # ---------------------------------------------------------- prefill ---
    if args.only != "decode":
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        Sf = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
        ws = kda.workspace(B, T, L, H, D, D, torch.bfloat16, CHUNK, device=dev)
        launches = kda.kda_forward_launches(B, T, L, H, D, D, kda.KDA_BF16, CHUNK)

        def fwd():
            kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], num_seqs=B,
                        chunk=CHUNK, o=o, S_final=Sf, workspace=ws, stream=stream)

        for _ in range(args.warmup):
            fwd()
        torch.cuda.synchronize()
        assert kda.check_device_error(ws) == kda.KDA_OK

        with ClockSampler(local) as clk:
            barrier()
            torch.cuda.synchronize()
            clk.mark()
            e0.record(stream)
            for _ in range(args.steps):
                fwd()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            ms_local = e0.elapsed_time(e1) / args.steps
        ms = rank_max(ms_local)
        out["clocks"] = clk.summary()
        out["ms"] = ms
        out["value"] = weak_scaling_value(T, world, ms)
        out["launches"] = launches * args.steps

        fwd_bytes = alg_bytes_prefill(T)
        fwd_flops = alg_flops(T)
        achieved = fwd_bytes / (ms_local / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                    "frac": achieved / pk["hbm"], "traffic": recorded_traffic("forward"),
                    "kernel": "kda_forward (one call: all %d launches)" % launches,
                    "peak_source": pk["src"],
                    "tensor_flops_frac": fwd_flops / (ms_local / 1e3) / 1e12 / pk["bf16"],
                    "roofline_time_us": max(fwd_bytes / pk["hbm"] / 1e3,
                                            fwd_flops / pk["bf16"] / 1e6)}
        roofline["frac_of_roofline_time"] = roofline["roofline_time_us"] / (ms_local * 1e3)
        out["roofline"] = roofline

        # ---------------------------------------------------------- e2e ---
        # Same metric through the public API with pinned host buffers: every
        # step copies its inputs in and reads o and S_final back inside the
        # timed region.  Steps are pipelined over three streams with two sets
        # of device buffers, as a serving loop would run them: the inputs of
        # step i+1 go in and the outputs of step i-1 come out while step i
        # computes (PCIe carries both directions at once).
        host = {k: inp[k].pin_memory() for k in ("q", "k", "v", "z", "beta", "A")}
        o_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        S_h = [torch.empty(Sf.shape, dtype=Sf.dtype).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_h[0].numel() * o_h[0].element_size() + S_h[0].numel() * S_h[0].element_size()
        dset = [d, {k_: torch.empty_like(d[k_]) for k_ in host}]
        o_d, S_d = [o, torch.empty_like(o)], [Sf, torch.empty_like(Sf)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

        def e2e_step(i):
            b = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])  # step i-2 has read this input set
                for k_, t in host.items():
                    dset[b][k_].copy_(t, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])     # step i-2's outputs have been read out
            x = dset[b]
            kda.forward(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], num_seqs=B,
                        chunk=CHUNK, o=o_d[b], S_final=S_d[b], workspace=ws, stream=stream)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                o_h[b].copy_(o_d[b], non_blocking=True)
                S_h[b].copy_(S_d[b], non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e2_0, e2_1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2_0.record(s_in)
        n_e2e = max(10, min(args.steps, 20))
        for i in range(n_e2e):
            e2e_step(i)
        e2_1.record(s_out)
        torch.cuda.synchronize()
        assert kda.check_device_error(ws) == kda.KDA_OK
        ms_e2e = rank_max(e2_0.elapsed_time(e2_1) / n_e2e)
        out["e2e"] = {"value": weak_scaling_value(T, world, ms_e2e), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
                      "pipelined": "three streams, two buffer sets: H2D of step i+1 and D2H "
                                   "of step i-1 overlap step i"}
        del dset[1], o_d[1], S_d[1]

        # ----------------------------------------------------- variants ---
        # The same workload through the entry points that add the output
        # epilogue and sparse state checkpoints; each is timed like the main
        # step and reported beside it with the bytes it adds.
        r_gate, w_gain = synth.out_gate_inputs(T, H, D, seed=5)
        r_gate, w_gain = r_gate.to(dev), w_gain.to(dev)
        interval = 4096
        ck = torch.empty((B, H, L // interval, D, D), dtype=torch.float32, device=dev)

        def fwd_norm_gate():
            kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], r_gate,
                                  norm_weight=w_gain, eps=1e-6, num_seqs=B, chunk=CHUNK, o=o,
                                  S_final=Sf, workspace=ws, stream=stream)

        def fwd_ckpt():
            kda.forward_checkpoints(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], interval,
                                    num_seqs=B, chunk=CHUNK, o=o, S_final=Sf, S_ckpt=ck,
                                    workspace=ws, stream=stream)

        cp_ws = torch.empty(kda.kda_cp_workspace_size(B, T, L, H, D, D, kda.KDA_BF16, CHUNK),
                            dtype=torch.uint8, device=dev)

        def fwd_cp():  # a context-parallel rank's two passes on one shard (the whole sequence)
            _, _, shard = kda.cp_local(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"],
                                       num_seqs=B, chunk=CHUNK, workspace=cp_ws, stream=stream)
            kda.cp_finish(shard, None, o=o, S_final=Sf, stream=stream)

        g_head = synth.scalar_gate(T, H, seed=7).to(dev)

        def fwd_scalar():  # the Gated DeltaNet case: one log-decay per token and head, no z
            kda.forward_scalar_gate(d["q"], d["k"], d["v"], g_head, d["beta"], num_seqs=B,
                                    chunk=CHUNK, o=o, S_final=Sf, workspace=ws, stream=stream)

        ci = {k_: t.to(dev) for k_, t in synth.conv_inputs(T, H, D, D, 4, seed=8).items()}
        conv_ws = torch.empty(kda.kda_forward_conv_workspace_size(B, T, L, H, D, D, kda.KDA_BF16,
                                                                  CHUNK),
                              dtype=torch.uint8, device=dev)

        def fwd_conv():  # input prologue (width-4 short convolution + Swish) fused into the operator
            kda.forward_conv(ci["x_q"], ci["x_k"], ci["x_v"], ci["w_q"], ci["w_k"], ci["w_v"],
                             d["z"], d["A"], d["beta"], num_seqs=B, chunk=CHUNK, o=o,
                             S_final=Sf, workspace=conv_ws, stream=stream)

        out["variants"] = {}
        n_var = max(3, min(args.steps, 20))
        for name, fn, extra in (
                ("norm_gate", fwd_norm_gate, T * H * D * 2 + D * 4),
                ("checkpoints_every_%d" % interval, fwd_ckpt, ck.numel() * 4),
                ("cp_local_and_finish", fwd_cp, 0),
                ("scalar_gate", fwd_scalar, T * H * 4 - T * H * D * 2),
                ("conv_prologue_width4", fwd_conv, 3 * H * D * 4 * 4)):  # + the taps
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            barrier()
            e0.record(stream)
            for _ in range(n_var):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms_v = e0.elapsed_time(e1) / n_var
            wsv = cp_ws if fn is fwd_cp else conv_ws if fn is fwd_conv else ws
            assert kda.check_device_error(wsv) == kda.KDA_OK
            ms_v = rank_max(ms_v)
            out["variants"][name] = {
                "ms_per_step": ms_v, "value": weak_scaling_value(T, world, ms_v),
                "unit": "tokens/s", "steps": n_var, "extra_alg_bytes": extra,
                "achieved_gbs": (fwd_bytes + extra) / (ms_v / 1e3) / 1e9}
        del ws, cp_ws, conv_ws, ci
        torch.cuda.empty_cache()
        if not args.no_configs:
            out["configs"] = time_configs(dev, stream, pk, world, rank_max, barrier, args.warmup,
                                          log)

    # ----------------------------------------------------------- decode ---
    if args.only != "prefill":
        A_dec, S_dec0 = synth.decode_state(DEC_B, H, D, D)
        S_dec = S_dec0.to(dev)
        A_dec = A_dec.to(dev)
        pool = [{k: t.to(dev) for k, t in synth.decode_token(s, DEC_B, H, D, D).items()}
                for s in range(8)]
        o_dec = torch.empty((DEC_B, H, D), dtype=torch.bfloat16, device=dev)

        def dec(s):
            tk = pool[s % len(pool)]
            kda.decode_step(tk["q"], tk["k"], tk["v"], tk["z"], A_dec, tk["beta"], S_dec,
                            o=o_dec, stream=stream)

        for s in range(10):
            dec(s)
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for s in range(args.decode_steps):
            dec(s)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_dec_local = e0.elapsed_time(e1) / args.decode_steps
        ms_dec = rank_max(ms_dec_local)
        # the decode step with the output epilogue fused in
        r_dec, w_dec = synth.out_gate_inputs(DEC_B, H, D, seed=6)
        r_dec, w_dec = r_dec.to(dev), w_dec.to(dev)

        def dec_ng(s):
            tk = pool[s % len(pool)]
            kda.decode_step_norm_gate(tk["q"], tk["k"], tk["v"], tk["z"], A_dec, tk["beta"],
                                      S_dec, r_dec, norm_weight=w_dec, eps=1e-6, o=o_dec,
                                      stream=stream)

        n_ng = max(10, args.decode_steps // 5)
        for s in range(10):
            dec_ng(s)
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for s in range(n_ng):
            dec_ng(s)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_ng = rank_max(e0.elapsed_time(e1) / n_ng)
        dec_bytes = alg_bytes_decode()
        dec_ach = dec_bytes / (ms_dec_local / 1e3) / 1e9
        out["decode"] = {
            "value": world * 1e3 / ms_dec, "unit": "steps/s", "ms_per_step": ms_dec,
            "tokens_per_s": world * DEC_B * 1e3 / ms_dec, "steps": args.decode_steps,
            "config": {"B": DEC_B, "H": H, "dk": D, "dv": D, "dtype": "bf16",
                       "state": "fp32 in place (268 MB, exceeds L2)"},
            "gpu_launches": args.decode_steps,
            "norm_gate": {"ms_per_step": ms_ng, "steps": n_ng,
                          "extra_alg_bytes": DEC_B * H * D * 2 + D * 4},
            "roofline": {"bound": "hbm", "achieved": dec_ach, "peak": pk["hbm"],
                         "unit": "GB/s", "frac": dec_ach / pk["hbm"],
                         "traffic": recorded_traffic("decode"),
                         "kernel": "decode_step_kernel", "peak_source": pk["src"]}}

    # ------------------------------------------------------ CPU baseline ---
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok = min(T, 16384)
        dt_cpu, cores = oracle_baseline(inp, n_tok)
        cpu = {"value": n_tok / dt_cpu, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {n_tok} tokens x {H} heads of the same workload (float64)"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": out["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": out["ms"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"KDA fwd long: B={B} H={H} L={L} dk=dv={D}, bf16 inputs, "
                               f"fp32 state, chunk {CHUNK}, S0=0", "B": B, "H": H, "L": L,
                   "dk": D, "dv": D, "chunk": CHUNK,
                   "arithmetic": "bf16 tensor-core operands with fp32 accumulation; gate, "
                                 "cumulative decay, norms, inverse and state in fp32",
                   "l2": "inputs exceed L2 (q,k,v,z,o = %.0f MB per step)" % (
                       T * H * D * 2 * 5 / 1e6),
                   "parallelism": f"weak x{world} (independent problems per rank)"},
        "roofline": out["roofline"], "cpu_baseline": cpu, "e2e": out["e2e"],
        "gpu_launches": out["launches"], "clocks": out["clocks"], "decode": out["decode"],
        "variants": out["variants"], "configs": out["configs"],
    }), flush=True)


if __name__ == "__main__":
    main()
