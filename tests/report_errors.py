"""Prints the errors of the CUDA path against the float64 oracle for every
workload configuration and entry point (max-abs and relative L2 of o / y and
of the final state).  Needs a GPU; run from the repository root:

    python tests/report_errors.py

The parity tests assert the bars; this script reports the measured margins."""
import os
import sys
import time

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from gated_delta_rule_98_b200 import kda, synth  # noqa: E402
from kda_testutil import f64, gpu_forward, oracle_forward, rel_l2, to_cuda  # noqa: E402


def line(name, o, o_ref, S=None, S_ref=None, t0=None):
    og = f64(o)
    msg = f"{name:44s} o max-abs {np.abs(og - o_ref).max():.3e} rel-L2 {rel_l2(og, o_ref):.3e}"
    if S is not None:
        Sg = f64(S)
        msg += f" | S max-abs {np.abs(Sg - S_ref).max():.3e} rel-L2 {rel_l2(Sg, S_ref):.3e}"
    if t0 is not None:
        msg += f"  ({time.time() - t0:.1f} s)"
    print(msg, flush=True)


def workloads():
    for name in ("tiny", "bf16", "varlen", "long"):
        t0 = time.time()
        inp = synth.workload(name)
        o, S = gpu_forward(inp, chunk=inp.get("chunk", 64))
        o_r, S_r = oracle_forward(inp)
        line(f"kda_forward {name}", o, o_r, S, S_r, t0)


def epilogue():
    from oracle import epilogue as ep
    for T, H, ns in ((1024, 4, 1), (8 * 192, 16, 8)):
        inp = synth.draw(T, H, 128, 128, seed=50 + H, dtype="bf16", num_seqs=ns, s0_std=0.02)
        inp["num_seqs"] = ns
        r, w = synth.out_gate_inputs(T, H, 128, seed=51)
        d = to_cuda(inp)
        y, S = kda.forward_norm_gate(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"],
                                     r.cuda(), norm_weight=w.cuda(), eps=1e-6, S0=d["S0"],
                                     num_seqs=ns, chunk=64)
        torch.cuda.synchronize()
        o_r, S_r = oracle_forward(inp)
        y_r = ep.norm_gate(o_r, f64(r), f64(w), eps=1e-6)
        line(f"kda_forward_norm_gate y T={T} H={H} N={ns}", y, y_r, S, S_r)
        # per-row relative error of y (one row = one token and head, dv values),
        # against the row's o norm relative to the median o row norm
        yg = f64(y)
        row_err = np.linalg.norm(yg - y_r, axis=-1) / np.maximum(np.linalg.norm(y_r, axis=-1), 1e-30)
        o_norm = np.linalg.norm(o_r, axis=-1)
        rel_norm = o_norm / np.median(o_norm)
        shares = ", ".join(f">{t:g}: {100 * np.mean(row_err > t):.2f}%" for t in (1e-3, 5e-3, 1e-2, 5e-2, 1e-1))
        low = row_err[rel_norm < 0.1]
        print(f"    y row errors: median {np.median(row_err):.2e}, p99 {np.quantile(row_err, 0.99):.2e}, "
              f"max {row_err.max():.2e}; rows {shares}; rows with |o| < 0.1 x median: "
              f"{100 * np.mean(rel_norm < 0.1):.2f}% of rows, their median error "
              f"{(np.median(low) if low.size else 0):.2e}", flush=True)


def prologue():
    from oracle import prologue as pr, ref
    cases = ((1024, 4, None, 1, 81), (8 * 192, 16, None, 8, 82),
             (sum([300, 0, 3, 411, 64]), 4, [300, 0, 3, 411, 64], 5, 83))
    for T, H, lens, ns, seed in cases:
        inp = synth.draw(T, H, 128, 128, seed=seed, dtype="bf16", num_seqs=ns, s0_std=0.02)
        ci = synth.conv_inputs(T, H, 128, 128, 4, seed=seed + 1)
        cu = synth.cu_from_lengths(lens) if lens else None
        d, dc = to_cuda(inp), to_cuda(ci)
        o, S = kda.forward_conv(dc["x_q"], dc["x_k"], dc["x_v"], dc["w_q"], dc["w_k"], dc["w_v"],
                                d["z"], d["A"], d["beta"], S0=d["S0"],
                                cu_seqlens=None if cu is None else cu.cuda(), num_seqs=ns,
                                max_seqlen=max(lens) if lens else T // ns, chunk=64)
        torch.cuda.synchronize()
        kw = dict(cu_seqlens=None if cu is None else cu.numpy(), num_seqs=ns)
        q = pr.short_conv_swish(ci["x_q"], ci["w_q"], **kw)
        k = pr.short_conv_swish(ci["x_k"], ci["w_k"], **kw)
        v = pr.short_conv_swish(ci["x_v"], ci["w_v"], **kw)
        o_r, S_r = ref.forward(q, k, v, inp["beta"], z=inp["z"], A=inp["A"], S0=inp["S0"], **kw)
        line(f"kda_forward_conv T={T} H={H} N={ns}", o, o_r, S, S_r)


def decode_conv(steps=120, width=4):
    from oracle import prologue as pr, ref
    B, H, D = 3, 2, 128
    T = B * steps
    ci = synth.conv_inputs(T, H, D, D, width, seed=140 + width)
    inp = synth.draw(T, H, D, D, seed=141 + width, dtype="bf16", num_seqs=B, s0_std=0.05)
    q = pr.short_conv_swish(ci["x_q"], ci["w_q"], num_seqs=B)
    k = pr.short_conv_swish(ci["x_k"], ci["w_k"], num_seqs=B)
    v = pr.short_conv_swish(ci["x_v"], ci["w_v"], num_seqs=B)
    at = lambda x, t: x.reshape(B, steps, *x.shape[1:])[:, t]
    w = {key: ci[key].cuda() for key in ("w_q", "w_k", "w_v")}
    state = kda.conv_state_zeros(B, H, D, D, width, torch.bfloat16)
    S, A, S_ref = inp["S0"].cuda(), inp["A"].cuda(), f64(inp["S0"])
    outs, refs = [], []
    for t in range(steps):
        outs.append(kda.decode_step_conv(at(ci["x_q"], t).cuda(), at(ci["x_k"], t).cuda(),
                                         at(ci["x_v"], t).cuda(), w["w_q"], w["w_k"], w["w_v"],
                                         state, at(inp["z"], t).cuda(), A,
                                         at(inp["beta"], t).cuda(), S))
        o_r, S_ref = ref.decode_step(at(q, t), at(k, t), at(v, t), f64(at(inp["beta"], t)),
                                     S_ref, z=f64(at(inp["z"], t)), A=f64(inp["A"]))
        refs.append(o_r)
    torch.cuda.synchronize()
    line(f"kda_decode_step_conv {steps} steps B={B} H={H}", torch.stack(outs, 1),
         np.stack(refs, 1), S, S_ref)


if __name__ == "__main__":
    workloads()
    epilogue()
    prologue()
    decode_conv()
