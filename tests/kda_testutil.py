"""Shared helpers of the KDA tests: tolerances, oracle runs, GPU runs."""
import numpy as np
import torch

# Tolerances of the operator's acceptance bar: fp32 inputs max-abs 1e-4;
# bf16 inputs (fp32 state) max-abs 2e-2 and relative L2 5e-3.  Both apply to
# o and to the final states.
TOL_F32_ABS = 1e-4
TOL_BF16_ABS = 2e-2
TOL_BF16_REL = 5e-3


def f64(t):
    return t.detach().cpu().double().numpy()


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def assert_close(got, want, dtype, what=""):
    """got: GPU result (torch, any dtype); want: float64 numpy oracle result."""
    g = f64(got)
    assert g.shape == want.shape, (what, g.shape, want.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = np.abs(g - want).max() if g.size else 0.0
    if dtype == torch.float32:
        assert err <= TOL_F32_ABS, f"{what}: max-abs {err:.3e} > {TOL_F32_ABS}"
    else:
        rel = rel_l2(g, want) if g.size else 0.0
        assert err <= TOL_BF16_ABS, f"{what}: max-abs {err:.3e} > {TOL_BF16_ABS}"
        assert rel <= TOL_BF16_REL, f"{what}: rel-L2 {rel:.3e} > {TOL_BF16_REL}"
    return err


def oracle_forward(inp, g=None, heads=None, threads=None):
    """Float64 oracle on the same (rounded) inputs.  ``heads`` restricts the
    run to a subset of heads (every head is an independent recurrence)."""
    from oracle import ref
    sel = (lambda t: t) if heads is None else (lambda t: t[:, heads])
    q, k, v, beta = sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["beta"])
    S0 = inp.get("S0")
    if S0 is not None and heads is not None:
        S0 = S0[:, heads]
    cu = inp.get("cu_seqlens")
    kw = dict(S0=S0, cu_seqlens=None if cu is None else cu.numpy(),
              num_seqs=inp.get("num_seqs", 1), threads=threads)
    if g is not None:
        return ref.forward(q, k, v, beta, g=sel(g), **kw)
    A = inp["A"] if heads is None else inp["A"][heads]
    return ref.forward(q, k, v, beta, z=sel(inp["z"]), A=A, **kw)


def to_cuda(inp):
    out = {}
    for key, val in inp.items():
        out[key] = val.cuda() if isinstance(val, torch.Tensor) else val
    return out


def max_len_of(inp):
    cu = inp.get("cu_seqlens")
    T = inp["q"].shape[0]
    if cu is None:
        return T // inp.get("num_seqs", 1)
    c = cu.cpu().numpy()
    return int(np.max(np.diff(c))) if len(c) > 1 else 0


def gpu_forward(inp, chunk=64, g=None, S0="inp", **kw):
    from gated_delta_rule_98_b200 import kda
    d = to_cuda(inp)
    s0 = d.get("S0") if isinstance(S0, str) else S0
    common = dict(S0=s0, cu_seqlens=d.get("cu_seqlens"), num_seqs=inp.get("num_seqs", 1),
                  max_seqlen=max_len_of(inp), chunk=chunk, **kw)
    if g is not None:
        o, S = kda.forward_g(d["q"], d["k"], d["v"], g.cuda(), d["beta"], **common)
    else:
        o, S = kda.forward(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], **common)
    torch.cuda.synchronize()
    return o, S
