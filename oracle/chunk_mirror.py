"""Chunkwise (WY / UT-transform) form of KDA in numpy float64.

TEST INFRASTRUCTURE ONLY.  This is not the oracle (``ref`` is); it restates,
step by step and in float64, the chunk algorithm that the GPU kernels run, so
that a kernel bug can be localised to one intermediate (A_kk, T, W, U~, U, O).
Its agreement with ``ref`` to ~1e-12 pins the chunk algebra below, which the
pages describe only in prose (Kimi Linear summary, §3.1 "Hardware-Efficient
Chunkwise Algorithm", §3.2, Appendix C; Kimi K3 architecture summary on the
16-token sub-tiles).

Derivation (from the recurrence, decay first).  For a chunk of n_c tokens
entering with state S, let Gam_r = sum_{s<=r} g_s (chunk-local, inclusive),
gam_r = exp(Gam_r).  Writing S_r = Diag(gam_r) S + sum_{i<=r}
Diag(gam_r/gam_i) k_i u_i^T and matching the per-token update gives

    A_kk[r,i] = beta_r sum_j k_rj k_ij exp(Gam_rj - Gam_ij)       (i <  r)
    A_qk[r,i] =        sum_j q_rj k_ij exp(Gam_rj - Gam_ij)       (i <= r)
    T         = (I + A_kk)^{-1}                 unit lower-triangular
    W         = T Diag(beta) (K * exp(Gam))      U~ = T Diag(beta) V
    U         = U~ - W S
    O         = (Q * exp(Gam)) S + A_qk U
    S_next    = Diag(exp(Gam_last)) S + (K * exp(Gam_last - Gam))^T U

Sub-tiles of 16 tokens keep every exponent a dense product can see bounded:
for row sub-tile b with reference rho_b = Gam of the token before it (0 for the
first), the row factor exp(Gam_r - rho_b) lies in [e^-80, 1] (16 tokens x
g >= -5) and the column factor exp(rho_b - Gam_i) is <= 1 for earlier
sub-tiles and < e^80 on the diagonal one.  T is formed by forward substitution
inside each 16x16 diagonal block, then block rows are combined as
T_ba = -T_bb sum_{a<=c<b} A_bc T_ca.
"""
from __future__ import annotations

import numpy as np

SUB = 16


def _unit(x, eps=1e-6):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def _gate(z, A):
    return -5.0 / (1.0 + np.exp(-np.exp(A) * z))


def forward_substitution_inverse(L):
    """(I + L)^{-1} for strictly lower-triangular L, one row at a time."""
    n = L.shape[0]
    X = np.zeros((n, n))
    for r in range(n):
        X[r, r] = 1.0
        for i in range(r):
            X[r, :] -= L[r, i] * X[i, :]
    return X


def intra_chunk_products(q, k, Gam, beta):
    """A_kk (strictly lower, rows scaled by beta) and A_qk (lower incl. diag)
    assembled from 16x16 blocks with per-row-sub-tile reference rho_b."""
    n = q.shape[0]
    Akk = np.zeros((n, n))
    Aqk = np.zeros((n, n))
    nb = (n + SUB - 1) // SUB
    for b in range(nb):
        rb = slice(b * SUB, min(n, (b + 1) * SUB))
        rho = Gam[b * SUB - 1] if b > 0 else np.zeros(Gam.shape[1])
        row_k = k[rb] * np.exp(Gam[rb] - rho)
        row_q = q[rb] * np.exp(Gam[rb] - rho)
        for a in range(b + 1):
            ra = slice(a * SUB, min(n, (a + 1) * SUB))
            col_k = k[ra] * np.exp(rho - Gam[ra])
            Akk[rb, ra] = row_k @ col_k.T
            Aqk[rb, ra] = row_q @ col_k.T
    Akk = np.tril(Akk, -1) * beta[:, None]
    Aqk = np.tril(Aqk, 0)
    return Akk, Aqk


def blocked_unit_lower_inverse(Akk):
    """T = (I + Akk)^{-1}: 16x16 diagonal blocks by forward substitution, then
    T_ba = -T_bb sum_{a<=c<b} A_bc T_ca for the blocks below the diagonal."""
    n = Akk.shape[0]
    nb = (n + SUB - 1) // SUB
    sl = [slice(b * SUB, min(n, (b + 1) * SUB)) for b in range(nb)]
    T = np.zeros((n, n))
    for b in range(nb):
        T[sl[b], sl[b]] = forward_substitution_inverse(Akk[sl[b], sl[b]])
    for b in range(nb):
        for a in range(b - 1, -1, -1):
            acc = np.zeros((sl[b].stop - sl[b].start, sl[a].stop - sl[a].start))
            for c in range(a, b):
                acc += Akk[sl[b], sl[c]] @ T[sl[c], sl[a]]
            T[sl[b], sl[a]] = -T[sl[b], sl[b]] @ acc
    return T


def chunk_step(S, q, k, v, g, beta, trace=None):
    """Advance state S over one chunk (n_c <= C tokens). Returns (O, S_next)."""
    Gam = np.cumsum(g, axis=0)
    Akk, Aqk = intra_chunk_products(q, k, Gam, beta)
    T = blocked_unit_lower_inverse(Akk)
    W = T @ (beta[:, None] * k * np.exp(Gam))
    Ut = T @ (beta[:, None] * v)
    U = Ut - W @ S
    O = (q * np.exp(Gam)) @ S + Aqk @ U
    Snext = np.exp(Gam[-1])[:, None] * S + (k * np.exp(Gam[-1] - Gam)).T @ U
    if trace is not None:
        trace.append(dict(Gam=Gam, Akk=Akk, Aqk=Aqk, T=T, W=W, Ut=Ut, U=U, O=O,
                          S_in=S.copy(), S_out=Snext.copy()))
    return O, Snext


def forward(q, k, v, beta, *, z=None, A=None, g=None, S0=None, cu_seqlens=None,
            chunk=64, trace=None):
    """Packed, multi-head chunkwise forward; same conventions as ``ref.forward``.
    The chunk grid restarts at every sequence start; the last chunk of a
    sequence may be partial."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    T_, H, dk = q.shape
    dv = v.shape[-1]
    if g is None:
        g = _gate(np.asarray(z, np.float64), np.asarray(A, np.float64)[None, :, None])
    g = np.asarray(g, np.float64)
    cu = np.array([0, T_]) if cu_seqlens is None else np.asarray(cu_seqlens, np.int64)
    N = len(cu) - 1
    o = np.zeros((T_, H, dv))
    Sf = np.zeros((N, H, dk, dv))
    qh = _unit(q)
    kh = _unit(k)
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[n, h], np.float64)
            for c0 in range(a, b, chunk):
                c1 = min(b, c0 + chunk)
                O, S = chunk_step(S, qh[c0:c1, h], kh[c0:c1, h], v[c0:c1, h],
                                  g[c0:c1, h], beta[c0:c1, h], trace)
                o[c0:c1, h] = O
            Sf[n, h] = S
    return o, Sf
