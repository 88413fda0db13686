"""KDA context parallelism: one long sequence split over the ranks of a
process group, shard r (in token order) on rank r.

Kimi K3 architecture summary, infrastructure section: KDA context parallelism
computes the local state updates on each rank and merges them with a prefix
scan over a fixed-size all-gather.  Because the recurrence is affine in the
state, shard r acts on the state entering it as S_after = M_r S_before + N_r.
Each rank

  1. computes (M_r, N_r) of its shard (``kda.cp_local``; the chunk preparation
     stays in the shard's workspace),
  2. all-gathers the packed [M_r | N_r] of every rank in one collective of a
     fixed size (H x dk x (dk + dv) fp32 per sequence),
  3. folds S_in(r) = M_{r-1}(... (M_0 S0 + N_0) ...) + N_{r-1} in rank order
     (``kda.state_compose``, one launch per earlier rank), and
  4. runs its shard's state pass from S_in(r) (``kda.cp_finish``).

The collective is the only exchange; every step of the arithmetic runs in the
library's kernels.  ``ops`` replaces those per-rank steps (the tests drive the
collective logic on CPU ranks with their own implementation).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class _KdaOps:
    """The per-rank steps on the GPU, through the C ABI."""

    def local(self, q, k, v, z, A, beta, cu_seqlens, max_seqlen, chunk):
        from . import kda
        return kda.cp_local(q, k, v, z, A, beta, cu_seqlens=cu_seqlens,
                            num_seqs=1 if cu_seqlens is None else None, max_seqlen=max_seqlen,
                            chunk=chunk)

    def compose(self, M, N, S):
        from . import kda
        return kda.state_compose(M, N, S)

    def finish(self, shard, S_in):
        from . import kda
        return kda.cp_finish(shard, S_in)


def context_parallel_forward(q, k, v, z, A, beta, *, S0=None, cu_seqlens=None, max_seqlen=None,
                             chunk=64, group=None, ops=None, events=None):
    """KDA prefill of this rank's shard of the sequences split over ``group``.

    q, k, z [T_r,H,dk], v [T_r,H,dv], beta [T_r,H]: this rank's tokens (the
    same sequences on every rank, each rank holding the next contiguous piece
    of each); S0 [N,H,dk,dv] the sequences' initial states (read on every rank,
    used by rank 0's fold); cu_seqlens the shard's own offsets.  ``events``,
    a pair of CUDA events, if given, is recorded around the all-gather (its
    share of the call).  Returns (o [T_r,H,dv], S_after [N,H,dk,dv]): on the
    last rank S_after is the sequences' final state.
    """
    ops = ops or _KdaOps()
    alone = not dist.is_initialized()  # one rank without a process group
    rank = 0 if alone else dist.get_rank(group)
    world = 1 if alone else dist.get_world_size(group)
    M, N, shard = ops.local(q, k, v, z, A, beta, cu_seqlens, max_seqlen, chunk)
    dk = M.shape[-1]
    packed = torch.cat([M, N], dim=-1).contiguous()          # [N,H,dk,dk+dv]
    gathered = [torch.empty_like(packed) for _ in range(world)]
    if events is not None:
        events[0].record()
    if world > 1:
        dist.all_gather(gathered, packed, group=group)
    else:
        gathered[0] = packed
    if events is not None:
        events[1].record()
    S = S0
    for j in range(rank):
        Mj = gathered[j][..., :dk].contiguous()
        Nj = gathered[j][..., dk:].contiguous()
        S = ops.compose(Mj, Nj, S)
    return ops.finish(shard, S)
