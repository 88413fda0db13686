"""Context parallelism in float64: the affine summary of a shard and the
prefix fold over shards.

TEST INFRASTRUCTURE ONLY.  Shares no code with the CUDA path.

Kimi K3 architecture summary, infrastructure section (KDA context
parallelism: local state updates per rank, merged by a prefix scan over an
all-gather); Kimi Linear summary §6.2 for the per-token transition
A_t = (I - beta_t k_t k_t^T) Diag(alpha_t).  A shard of tokens t = 1 .. L maps
the state entering it to S_after = M S_before + N with

    M = A_L ... A_2 A_1            (the product of the shard's transitions)
    N = the state the shard leaves when it starts from S = 0

and the state entering shard r is S_in(r) = M_{r-1} S_in(r-1) + N_{r-1},
S_in(0) = S0.
"""
from __future__ import annotations

import numpy as np

from . import brute, ref


def shard_transition(q, k, v, beta, z, A):
    """(M [H,dk,dk], N [H,dk,dv]) of one shard of one sequence, float64.
    q, k, z [L,H,dk]; v [L,H,dv]; beta [L,H]; A [H]."""
    q, k, v, beta, z = (ref._f64(x) for x in (q, k, v, beta, z))
    L, H, dk = k.shape
    g = brute.lower_bounded_gate(z, A)
    kh = brute.unit(k)
    M = np.zeros((H, dk, dk))
    for h in range(H):
        P = np.eye(dk)
        for t in range(L):
            P = brute.transition(np.exp(g[t, h]), beta[t, h], kh[t, h]) @ P
        M[h] = P
    _, N = ref.forward(q, k, v, beta, z=z, A=A, num_seqs=1)
    return M, N[0]


def compose(M, N, S):
    """M S + N per head (S None reads as zeros)."""
    return N.copy() if S is None else np.einsum("hij,hjk->hik", M, S) + N


def prefix_states(Ms, Ns, S0=None):
    """Incoming state of every shard: S_in(0) = S0, S_in(r+1) = M_r S_in(r) + N_r."""
    out = [S0]
    for M, N in zip(Ms[:-1], Ns[:-1]):
        out.append(compose(M, N, out[-1]))
    return out
