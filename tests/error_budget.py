"""Error budget of the tensor-core prefill on the CPU: where o's error against
the float64 oracle comes from.

The chunkwise algebra (Kimi Linear summary §3.1, with the 16-token sub-tiles
of the Kimi K3 architecture summary) is evaluated in float32 with each
operand rounding the tensor-core kernels apply switched on alone, all
together, or all but one:

  m1_kk     bf16 operands of A_kk (beta k E rows x key windows)
  m1_qr     bf16 q E rows of A_qk
  m1_qc     bf16 key windows of A_qk (off-diagonal 16 x 16 blocks)
  m1_qd     bf16 operands of A_qk's four diagonal 16 x 16 blocks
  slot_aqk  A_qk stored in f16
  m2_t      f16 T and beta k e^Gamma in W = T Diag(beta) (K e^Gamma)
  m2_v      bf16 T Diag(beta) and V in U~ = T Diag(beta) V
  slot      W, U~, Q', K' stored in f16
  chain_s   the f16 copy of S that multiplies [Q'; W]
  chain_u   U = U~ - W S rounded to f16
  out       o rounded to bf16

and, once each, with the chain products reassociated (see ``chunked``) and
with 128-token chunks.

Run from the repository root (CPU only, about a minute):

    python tests/error_budget.py

It measures four heads of the L=4096 bf16 workload, then the output
epilogue y = RMSNorm(o) * w * sigmoid(r) (Kimi Linear summary §4) on the
T=1024, H=4 case with a nonzero initial state, where y is formed from the
float32 o as the fused epilogue does.  The kernels' own figures for both
come from ``tests/report_errors.py`` on a GPU."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from gated_delta_rule_98_b200 import synth  # noqa: E402
from oracle import epilogue, ref  # noqa: E402


def bf16(x):
    """Round to bfloat16 (nearest, ties to even), kept in float32."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def f16(x):
    """Round to IEEE half (saturating at the largest finite value)."""
    return np.clip(np.asarray(x, np.float32), -65504, 65504).astype(np.float16).astype(np.float32)


def tf32(x):
    """Round to 10 explicit mantissa bits with the float32 exponent."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0xFFF + ((u >> 13) & 1)) >> 13) << 13
    return r.astype(np.uint32).view(np.float32)


def hi_lo(x):
    """A bf16 pair hi + lo (about 16 mantissa bits)."""
    hi = bf16(x)
    return hi + bf16(np.asarray(x, np.float32) - hi)


def exact(x):
    return np.asarray(x, np.float32)


GROUPS = ("m1_kk", "m1_qr", "m1_qc", "m1_qd", "slot_aqk", "m2_t", "m2_v", "slot", "chain_s",
          "chain_u", "out")
KERNEL = dict(m1_kk=bf16, m1_qr=bf16, m1_qc=bf16, m1_qd=bf16, slot_aqk=f16, m2_t=f16, m2_v=bf16,
              slot=f16, chain_s=f16, chain_u=f16, out=bf16)
NONE = {g: exact for g in GROUPS}
C, SUB = 64, 16


def prepare(inp, h, R, C=C):
    """The state-independent operands of every chunk (C tokens) of head h
    (what the chunk preparation writes to the chunk slots), with the
    roundings R."""
    q = inp["q"].float().numpy()[:, h]
    k = inp["k"].float().numpy()[:, h]
    v = inp["v"].float().numpy()[:, h]
    z = inp["z"].float().numpy()[:, h]
    beta = inp["beta"].float().numpy()[:, h]
    a_h = float(inp["A"][h])
    D = q.shape[-1]
    chunks = []
    for c0 in range(0, q.shape[0], C):
        qc, kc, vc, bc = q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], beta[c0:c0 + C]
        g = (-5.0 / (1.0 + np.exp(-np.exp(a_h) * z[c0:c0 + C]))).astype(np.float32)
        Gam = np.cumsum(g, axis=0, dtype=np.float32)
        kn = kc / np.sqrt((kc * kc).sum(-1, keepdims=True) + 1e-6)
        Akk = np.zeros((C, C), np.float32)
        Aqk = np.zeros((C, C), np.float32)
        for b in range(C // SUB):
            rb = slice(SUB * b, SUB * (b + 1))
            rho = Gam[SUB * b - 1] if b > 0 else np.zeros(D, np.float32)
            E = np.exp(Gam[rb] - rho)  # <= 1
            for a in range(b + 1):
                ra = slice(SUB * a, SUB * (a + 1))
                col = kn[ra] * np.exp(rho - Gam[ra])  # <= 1 for a < b, up to e^80 for a = b
                Akk[rb, ra] = R["m1_kk"](bc[rb, None] * kn[rb] * E) @ R["m1_kk"](col).T
                if a == b:
                    Aqk[rb, ra] = R["m1_qd"](qc[rb] * E) @ R["m1_qd"](col).T
                else:
                    Aqk[rb, ra] = R["m1_qr"](qc[rb] * E) @ R["m1_qc"](col).T
        Akk = np.tril(Akk, -1)
        Tm = np.tril(np.linalg.inv(np.eye(C, dtype=np.float32) + Akk).astype(np.float32))
        W = R["slot"](R["m2_t"](Tm) @ R["m2_t"](bc[:, None] * kn * np.exp(Gam)))
        chunks.append(dict(
            Y=np.concatenate([R["slot"](qc * np.exp(Gam)), W]),     # [Q'; W]
            Aqk=R["slot_aqk"](np.tril(Aqk, 0)),
            Ut=R["slot"](R["m2_v"](Tm * bc[None, :]) @ R["m2_v"](vc)),
            Kp=R["slot"](kn * np.exp(Gam[-1] - Gam)),              # K'
            gam=np.exp(Gam[-1]),
            iq=1.0 / np.sqrt((qc * qc).sum(-1, keepdims=True) + 1e-6)))
    return chunks


def chunked(inp, heads, R, S0=None, reassociated=False, C=C):
    """o [T, len(heads), dv] of the chunkwise form with the roundings R, from
    the initial states S0 [1, H, dk, dv] (zero when None).

    reassociated: each chunk's state product is formed from the state before
    the previous chunk, Y_{c+1} S_c = (Y_{c+1} Diag(gamma_c)) S_{c-1} +
    (Y_{c+1} K'_c^T) U_c, with both new factors rounded like the slot images
    (a schedule with one dependent product per chunk instead of two)."""
    dv = inp["v"].shape[-1]
    o = np.zeros((inp["q"].shape[0], len(heads), dv), np.float32)
    for hi, h in enumerate(heads):
        ch = prepare(inp, h, R, C)
        S = (np.zeros((inp["q"].shape[-1], dv), np.float32) if S0 is None
             else np.array(S0[0, h], np.float32))
        Dm = ch[0]["Y"] @ R["chain_s"](S)
        for c, x in enumerate(ch):
            if not reassociated:
                Dm = x["Y"] @ R["chain_s"](S)
            U = R["chain_u"](x["Ut"] - Dm[C:])
            o[c * C:(c + 1) * C, hi] = R["out"]((Dm[:C] + x["Aqk"] @ U) * x["iq"])
            if reassociated and c + 1 < len(ch):
                y = ch[c + 1]["Y"]
                Dm = (R["slot"](y * x["gam"][None, :]) @ R["chain_s"](S)
                      + R["slot"](y @ x["Kp"].T) @ U)
            S = x["gam"][:, None] * S + x["Kp"].T @ U
    return o


def main():
    inp = synth.workload("bf16")
    heads = [0, 5, 10, 15]
    d = {n: inp[n].double().numpy()[:, heads] for n in ("q", "k", "v", "beta", "z")}
    o_ref, _ = ref.forward(d["q"], d["k"], d["v"], d["beta"], z=d["z"],
                           A=inp["A"].double().numpy()[heads])

    def rel(R):
        o = chunked(inp, heads, R)
        return np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref)

    def show(name, R):
        print(f"{name:58s} o rel-L2 {rel(R):.3e}", flush=True)

    show("no rounding (float32 arithmetic)", NONE)
    show("every rounding of the kernels", KERNEL)
    for g in GROUPS:
        show(f"only {g}", {**NONE, g: KERNEL[g]})
    for g in GROUPS:
        show(f"all but {g}", {**KERNEL, g: exact})
    show("earlier kernel: slots and chain operands in bf16",
         {**KERNEL, "slot": bf16, "slot_aqk": bf16, "chain_s": bf16, "chain_u": bf16, "m2_t": bf16})
    show("only the S copy in bf16", {**NONE, "chain_s": bf16})
    show("kernel, A_qk diagonal blocks as hi + lo bf16 pairs", {**KERNEL, "m1_qd": hi_lo})
    show("kernel, A_qk diagonal blocks in tf32", {**KERNEL, "m1_qd": tf32})
    show("kernel, A_qk diagonal blocks in float32", {**KERNEL, "m1_qd": exact})
    show("kernel, A_qk diagonal blocks in float32, o in float32",
         {**KERNEL, "m1_qd": exact, "out": exact})
    for name, kw in (("kernel, reassociated chain schedule", dict(reassociated=True)),
                     ("kernel, 128-token chunks", dict(C=128))):
        o = chunked(inp, heads, KERNEL, **kw)
        print(f"{name:58s} o rel-L2 {np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref):.3e}",
              flush=True)

    # the output epilogue, from the float32 o
    T, H = 1024, 4
    e_inp = synth.draw(T, H, 128, 128, seed=50 + H, dtype="bf16", num_seqs=1, s0_std=0.02)
    r, w = synth.out_gate_inputs(T, H, 128, seed=51)
    d = {n: e_inp[n].double().numpy() for n in ("q", "k", "v", "beta", "z")}
    eo_ref, _ = ref.forward(d["q"], d["k"], d["v"], d["beta"], z=d["z"],
                            A=e_inp["A"].double().numpy(), S0=e_inp["S0"].double().numpy())
    y_ref = epilogue.norm_gate(eo_ref, r.double().numpy(), w.double().numpy(), eps=1e-6)
    rn, wn = r.float().numpy(), w.numpy()
    S0 = e_inp["S0"].numpy()
    for name, R in (("kernel", KERNEL), ("kernel, A_qk diagonal blocks as hi + lo pairs",
                                         {**KERNEL, "m1_qd": hi_lo})):
        o32 = chunked(e_inp, list(range(H)), {**R, "out": exact}, S0)
        y = bf16(o32 / np.sqrt(np.mean(o32 * o32, -1, keepdims=True) + 1e-6) * wn
                 / (1.0 + np.exp(-rn)))
        print(f"epilogue T={T} H={H}, {name:37s} y rel-L2 "
              f"{np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref):.3e}", flush=True)


if __name__ == "__main__":
    main()
