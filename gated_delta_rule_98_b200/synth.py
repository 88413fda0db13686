"""Seeded synthetic inputs for the KDA operator.

This module only draws random numbers and shapes them into the operator's
input layout; it holds none of the operator's arithmetic.  Both the CUDA path
(via the tests and the benchmark) and the float64 oracle consume exactly the
tensors it returns, so the two sides see bit-identical inputs (bf16 values are
widened exactly to float64 on the oracle side).

Recipe (numpy ``default_rng(seed)``, PCG64, draws in float64 in this order):
  q, k ~ N(0,1) [T,H,dk], each (token, head) row scaled to unit length
  v ~ N(0,1) [T,H,dv]
  beta = logistic(N(0,1)) [T,H]
  z ~ N(0,1) [T,H,dk]
  A ~ N(0,1) [H]                      (kept fp32)
  S0 ~ N(0, s0_std^2) [N,H,dk,dv]     (kept fp32; omitted when s0_std is None)
q, k, v, z, beta are then rounded to the compute dtype (round-to-nearest-even).

Output epilogue inputs (``out_gate_inputs``, numpy ``default_rng(seed)``):
  r ~ N(0,1) [T,H,dv]                 (gate logits; rounded to the compute dtype)
  w ~ U(0.5, 1.5) [dv]                (RMSNorm gain, fp32)
Input prologue (``conv_inputs``, ``default_rng(seed)``, in this order):
  x_q, x_k ~ N(0,1) [T,H,dk], x_v ~ N(0,1) [T,H,dv]   (rounded to the compute dtype)
  w_q, w_k ~ N(0,1/width) [H*dk,width], w_v ~ N(0,1/width) [H*dv,width]   (fp32)
Scalar (per token and head) log-decay (``scalar_gate``, ``default_rng(seed)``):
  alpha ~ U(e^-5, 1) [T,H], g = ln(alpha) fp32, in [-5, 0)

Workloads (sizes follow the operator's published benchmark settings):
  tiny      B=1 H=2  L=64    d=32  fp32 chunk 16  S0=0           seed 0
  bf16      B=1 H=16 L=4096  d=128 bf16 chunk 64  S0=0           seed 1
  long      B=1 H=16 L=65536 d=128 bf16 chunk 64  S0=0           seed 2
  varlen    T=32768 packed, lengths in [512,8192], H=32, d=128, bf16,
            S0 ~ N(0, 0.02^2)                                    seed 3
  decode    B=256 H=16 d=128 bf16, persistent S ~ N(0, 0.02^2),
            A and S from default_rng(4); step s from default_rng([4, s])
"""
from __future__ import annotations

import numpy as np
import torch

_DT = {"f32": torch.float32, "fp32": torch.float32, "float32": torch.float32,
       "bf16": torch.bfloat16, "bfloat16": torch.bfloat16}


def torch_dtype(dt):
    if isinstance(dt, torch.dtype):
        return dt
    return _DT[dt]


def _unit_rows(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def _cast(x, dtype):
    # torch's round-to-nearest-even conversion; both sides of every comparison
    # receive the rounded values, so the rounding path itself is immaterial.
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def draw(T, H, dk, dv, *, seed, dtype="bf16", num_seqs=1, s0_std=None, rng=None):
    """Inputs for T tokens (packed over ``num_seqs`` sequences) in the recipe's
    draw order.  Returns a dict of CPU torch tensors."""
    dtype = torch_dtype(dtype)
    rng = np.random.default_rng(seed) if rng is None else rng
    out = {}
    out["q"] = _cast(_unit_rows(rng.standard_normal((T, H, dk))), dtype)
    out["k"] = _cast(_unit_rows(rng.standard_normal((T, H, dk))), dtype)
    out["v"] = _cast(rng.standard_normal((T, H, dv)), dtype)
    out["beta"] = _cast(1.0 / (1.0 + np.exp(-rng.standard_normal((T, H)))), dtype)
    out["z"] = _cast(rng.standard_normal((T, H, dk)), dtype)
    out["A"] = torch.from_numpy(rng.standard_normal(H)).float()
    if s0_std is not None:
        out["S0"] = torch.from_numpy(
            rng.standard_normal((num_seqs, H, dk, dv)) * s0_std).float()
    else:
        out["S0"] = None
    return out


def out_gate_inputs(T, H, dv, *, seed, dtype="bf16"):
    """Gate input r [T,H,dv] (compute dtype) and gain w [dv] (fp32) for the
    output epilogue, drawn in that order."""
    rng = np.random.default_rng(seed)
    r = _cast(rng.standard_normal((T, H, dv)), torch_dtype(dtype))
    w = torch.from_numpy(rng.uniform(0.5, 1.5, dv)).float()
    return r, w


def conv_inputs(T, H, dk, dv, width, *, seed, dtype="bf16"):
    """Pre-convolution q, k, v and the depthwise taps of the input prologue."""
    rng = np.random.default_rng(seed)
    dt = torch_dtype(dtype)
    out = {}
    out["x_q"] = _cast(rng.standard_normal((T, H, dk)), dt)
    out["x_k"] = _cast(rng.standard_normal((T, H, dk)), dt)
    out["x_v"] = _cast(rng.standard_normal((T, H, dv)), dt)
    s = 1.0 / np.sqrt(width)
    out["w_q"] = torch.from_numpy(rng.standard_normal((H * dk, width)) * s).float()
    out["w_k"] = torch.from_numpy(rng.standard_normal((H * dk, width)) * s).float()
    out["w_v"] = torch.from_numpy(rng.standard_normal((H * dv, width)) * s).float()
    return out


def scalar_gate(T, H, *, seed):
    """One log-decay per token and head (Gated DeltaNet form), fp32 [T,H]:
    the log of a decay drawn uniformly from [e^-5, 1)."""
    rng = np.random.default_rng(seed)
    g = np.log(rng.uniform(np.exp(-5.0), 1.0, (T, H)))
    return torch.from_numpy(np.maximum(g, -5.0)).float()


def varlen_lengths(total=32768, lo=512, hi=8192, seed=3):
    """Sequence lengths in [lo, hi] summing to ``total``: draw uniformly from
    [lo, hi], never leaving a remainder below ``lo``; the last length is the
    remainder once it fits in [lo, hi]."""
    rng = np.random.default_rng(seed)
    lens = []
    rem = total
    while rem > hi:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, rem - lo)
        lens.append(L)
        rem -= L
    lens.append(rem)
    assert sum(lens) == total and all(lo <= L <= hi for L in lens)
    return lens


def cu_from_lengths(lens):
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    return torch.from_numpy(cu)


WORKLOADS = {
    "tiny":   dict(B=1, H=2, L=64, dk=32, dv=32, dtype="f32", chunk=16, seed=0, s0_std=None),
    "bf16":   dict(B=1, H=16, L=4096, dk=128, dv=128, dtype="bf16", chunk=64, seed=1, s0_std=None),
    "long":   dict(B=1, H=16, L=65536, dk=128, dv=128, dtype="bf16", chunk=64, seed=2, s0_std=None),
    "varlen": dict(T=32768, H=32, dk=128, dv=128, dtype="bf16", chunk=64, seed=3, s0_std=0.02),
    "decode": dict(B=256, H=16, dk=128, dv=128, dtype="bf16", seed=4, s0_std=0.02, steps=1000),
}


def workload(name, L=None):
    """Inputs for a named prefill workload.  ``L`` overrides the length of
    'long' (its sweep uses 2048, 8192, 32768, 65536)."""
    w = WORKLOADS[name]
    if name == "varlen":
        lens = varlen_lengths(w["T"], seed=w["seed"])
        inp = draw(w["T"], w["H"], w["dk"], w["dv"], seed=w["seed"], dtype=w["dtype"],
                   num_seqs=len(lens), s0_std=w["s0_std"])
        inp["cu_seqlens"] = cu_from_lengths(lens)
        inp["num_seqs"] = len(lens)
        inp["chunk"] = w["chunk"]
        return inp
    L = w["L"] if L is None else L
    inp = draw(w["B"] * L, w["H"], w["dk"], w["dv"], seed=w["seed"], dtype=w["dtype"],
               num_seqs=w["B"], s0_std=w["s0_std"])
    inp["cu_seqlens"] = None
    inp["num_seqs"] = w["B"]
    inp["chunk"] = w["chunk"]
    return inp


def decode_state(B=256, H=16, dk=128, dv=128, seed=4, s0_std=0.02):
    """(A [H] fp32, S [B,H,dk,dv] fp32) for the decode workload."""
    rng = np.random.default_rng(seed)
    A = torch.from_numpy(rng.standard_normal(H)).float()
    S = torch.from_numpy(rng.standard_normal((B, H, dk, dv)) * s0_std).float()
    return A, S


def decode_token(step, B=256, H=16, dk=128, dv=128, seed=4, dtype="bf16"):
    """Token inputs of decode step ``step``: q, k, v, beta, z (dtype)."""
    dtype = torch_dtype(dtype)
    rng = np.random.default_rng([seed, step])
    return {
        "q": _cast(_unit_rows(rng.standard_normal((B, H, dk))), dtype),
        "k": _cast(_unit_rows(rng.standard_normal((B, H, dk))), dtype),
        "v": _cast(rng.standard_normal((B, H, dv)), dtype),
        "beta": _cast(1.0 / (1.0 + np.exp(-rng.standard_normal((B, H)))), dtype),
        "z": _cast(rng.standard_normal((B, H, dk)), dtype),
    }
