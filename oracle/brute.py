"""Brute-force KDA by materialised transition products (numpy, float64).

TEST INFRASTRUCTURE ONLY.  Tiny sizes (L <= ~32, d <= ~8): the cost is
O(L^2 d^3).  Shares no code with ``ref`` or the CUDA path.

It follows two other views of the same operator that the pages give:

* Kimi Linear summary, §6.2 "Relation to DPLR": the per-token transition is
  the constrained DPLR matrix  A_t = Diag(alpha_t) - beta_t k_t k_t^T Diag(alpha_t).
* Kimi Linear summary, §6.1 (KDA as learnable position embeddings): the
  interaction between a past key i and the query at t is carried by the
  cumulative product of transitions between them,
  P_{t<-i} = A_t A_{t-1} ... A_{i+1}  (P_{t<-t} = I).

Unrolling S_t = A_t S_{t-1} + beta_t k_t v_t^T gives

    S_t   = P_{t<-0} S_0 + sum_{i<=t} P_{t<-i} beta_i k_i v_i^T
    o_t   = sum_{i<=t} Attn[t,i] v_i + (P_{t<-0} S_0)^T q_t,
    Attn[t,i] = beta_i q_t^T P_{t<-i} k_i     (causal, diagonal included).
"""
from __future__ import annotations

import numpy as np


def unit(x, eps=1e-6):
    """Rows scaled to unit length, x / sqrt(sum x^2 + eps)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def lower_bounded_gate(z, A, g_min=-5.0):
    """g = g_min * logistic(exp(A_h) z) for z [T,H,dk] and A [H]."""
    z = np.asarray(z, np.float64)
    s = np.exp(np.asarray(A, np.float64))[None, :, None] * z
    return g_min * (1.0 / (1.0 + np.exp(-s)))


def transition(alpha, beta, k):
    """Constrained DPLR transition Diag(alpha) - beta k k^T Diag(alpha)."""
    D = np.diag(alpha)
    return D - beta * np.outer(k, k) @ D


def single_head(q, k, v, g, beta, S0=None):
    """One sequence, one head.  q,k,g [L,dk]; v [L,dv]; beta [L]; S0 [dk,dv].

    Returns (o [L,dv], S_final [dk,dv], Attn [L,L])."""
    q = unit(q)
    k = unit(k)
    v = np.asarray(v, np.float64)
    L, dk = q.shape
    dv = v.shape[1]
    S0 = np.zeros((dk, dv)) if S0 is None else np.asarray(S0, np.float64)
    alpha = np.exp(np.asarray(g, np.float64))
    Amat = [transition(alpha[t], beta[t], k[t]) for t in range(L)]

    def P(t, i):  # product of transitions of tokens i+1..t (0-based: tokens i+1..t)
        M = np.eye(dk)
        for s in range(i + 1, t + 1):
            M = Amat[s] @ M
        return M

    attn = np.zeros((L, L))
    o = np.zeros((L, dv))
    for t in range(L):
        for i in range(t + 1):
            attn[t, i] = beta[i] * q[t] @ P(t, i) @ k[i]
        # the incoming state sees every transition of tokens 0..t
        P0 = np.eye(dk)
        for s in range(t + 1):
            P0 = Amat[s] @ P0
        o[t] = attn[t, : t + 1] @ v[: t + 1] + (P0 @ S0).T @ q[t]
    Sf = np.zeros((dk, dv))
    P0 = np.eye(dk)
    for s in range(L):
        P0 = Amat[s] @ P0
    Sf += P0 @ S0
    for i in range(L):
        Sf += P(L - 1, i) @ np.outer(beta[i] * k[i], v[i])
    return o, Sf, attn


def forward(q, k, v, beta, *, z=None, A=None, g=None, S0=None, cu_seqlens=None):
    """Packed multi-sequence, multi-head driver of ``single_head``.

    q,k,(z|g) [T,H,dk]; v [T,H,dv]; beta [T,H]; A [H]; S0 [N,H,dk,dv] or None;
    cu_seqlens [N+1] or None (one sequence)."""
    q = np.asarray(q, np.float64)
    T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    if g is None:
        g = lower_bounded_gate(z, A)
    g = np.asarray(g, np.float64)
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, np.int64)
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    Sf = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            s0 = None if S0 is None else np.asarray(S0, np.float64)[n, h]
            if b == a:
                Sf[n, h] = 0.0 if s0 is None else s0
                continue
            o[a:b, h], Sf[n, h], _ = single_head(q[a:b, h], np.asarray(k)[a:b, h],
                                                 np.asarray(v)[a:b, h], g[a:b, h],
                                                 np.asarray(beta, np.float64)[a:b, h], s0)
    return o, Sf
