"""Sequence-sharded attention over several GPUs: a ring of K/V shards and
the exact log-sum-exp merge.

Source: the briefgpt.xyz summary page of FlashAttention-2 (arXiv
2307.08691), entry "BurstAttention": attention distributed over devices
along the sequence, with communication reduced by organising it at both the
cluster and the device level.  Reading taken here (the entry gives no
algorithm): the sequence of length N is split into P contiguous shards, one
per rank; rank r holds Q_r, K_r, V_r.  In P steps the K/V shards travel
around the ring (rank r sends to r + 1 and receives from r - 1) while each
rank attends its queries to the shard it holds with the single-GPU kernel
(non-causal for an earlier shard, causal for its own, skipped for a later
one under the causal mask) and folds the partial (O, lse) into an fp32
accumulator:  lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s --
inside the kernel's epilogue (attn_fwd_merge: the first block writes the
accumulator, later ones merge into it, the last writes the bf16 result).
The result is exact attention for the rank's queries.  The exchange of the
next shard is started before the current step's compute, so the transfer
overlaps it.

Everything here is orchestration: every arithmetic step runs in the CUDA
library (attn_fwd_merge, or attn_fwd for a rank with one block) through
``GpuOps``; tests may pass other ops with the same method.
"""
from __future__ import annotations

from dataclasses import dataclass


def shard_plan(rank: int, world: int, causal: bool):
    """Per ring step t: (key shard held, how it is attended) with how one of
    "full", "causal", None (nothing: every key of the shard lies in the
    future of every query of this rank)."""
    plan = []
    for t in range(world):
        s = (rank - t) % world
        if s == rank:
            how = "causal" if causal else "full"
        elif s < rank or not causal:
            how = "full"
        else:
            how = None
        plan.append((s, how))
    return plan


class GpuOps:
    """The CUDA library's block attention with the fold in its epilogue (no
    fallback)."""

    def __init__(self):
        from . import attn
        self.attn = attn

    def block(self, q, k, v, causal: bool, scale: float, state: dict, i: int,
              n: int):
        """Block i of the n blocks this rank attends; returns (O, lse) after
        the last (i = n - 1), None before."""
        import torch
        if n == 1:
            return self.attn.attn_fwd(q, k, v, causal=causal, scale=scale)
        if i == 0:
            B, H, m, d = q.shape
            state["o"] = torch.empty((B, H, m, d), dtype=torch.float32, device=q.device)
            state["lse"] = torch.empty((B, H, m), dtype=torch.float32, device=q.device)
        mode = (self.attn.MERGE_FIRST if i == 0 else
                self.attn.MERGE_LAST if i == n - 1 else self.attn.MERGE_INTO)
        return self.attn.attn_fwd_merge(q, k, v, state["o"], state["lse"], mode,
                                        causal=causal, scale=scale)


@dataclass
class RingStats:
    steps: int = 0
    blocks: int = 0
    skipped: int = 0
    bytes_sent: int = 0


def ring_attention(q, k, v, causal: bool, scale: float, group=None, ops=None,
                   stats: RingStats | None = None):
    """Exact attention of this rank's queries q [B, H, n, d] over the whole
    sequence, whose K/V shards k, v [B, H, n, d] (this rank's) travel around
    the ring of `group` (torch.distributed; world 1 = no exchange).  Returns
    (O [B, H, n, d] bf16, lse [B, H, n] fp32) for this rank's queries."""
    import torch
    import torch.distributed as dist
    ops = ops or GpuOps()
    result = None
    world = dist.get_world_size(group) if (group is not None or dist.is_initialized()) else 1
    rank = dist.get_rank(group) if world > 1 else 0
    plan = shard_plan(rank, world, causal)
    nblocks = sum(how is not None for _, how in plan)
    kv = torch.stack([k, v]).contiguous()
    nxt = torch.empty_like(kv) if world > 1 else None
    state, done = {}, 0
    for t, (s, how) in enumerate(plan):
        reqs = []
        if world > 1 and t + 1 < world:
            # start passing the shard on (and receiving the next) before the
            # compute that uses it
            peer_to, peer_from = (rank + 1) % world, (rank - 1) % world
            reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, kv, peer_to, group),
                dist.P2POp(dist.irecv, nxt, peer_from, group)])
            if stats is not None:
                stats.bytes_sent += kv.numel() * kv.element_size()
        if how is not None:
            out = ops.block(q, kv[0], kv[1], how == "causal", scale, state, done,
                            nblocks)
            done += 1
            if done == nblocks:
                result = out
            if stats is not None:
                stats.blocks += 1
        elif stats is not None:
            stats.skipped += 1
        for r in reqs:
            r.wait()
        if reqs:
            kv, nxt = nxt, kv
        if stats is not None:
            stats.steps += 1
    return result


def shard(x, world: int):
    """The `world` contiguous sequence shards of x [B, H, N, d] (N divisible
    by world), each made contiguous: what rank r holds."""
    B, H, N, d = x.shape
    if N % world:
        raise ValueError("N must be a multiple of the number of shards")
    n = N // world
    return [x[:, :, r * n:(r + 1) * n].contiguous() for r in range(world)]


def ring_attention_emulated(qs, ks, vs, causal: bool, scale: float, ops=None,
                            stats: RingStats | None = None):
    """The ring algorithm of len(qs) ranks run one rank after another on one
    device; qs, ks, vs are the ranks' contiguous shards (see `shard`).  Rank
    r's step t attends its queries to key shard (r - t) mod P -- exactly the
    blocks the distributed run computes.  Returns the ranks' (O, lse) lists."""
    ops = ops or GpuOps()
    world = len(qs)
    outs, lses = [], []
    for r in range(world):
        plan = shard_plan(r, world, causal)
        nblocks = sum(how is not None for _, how in plan)
        state, done, result = {}, 0, None
        for s, how in plan:
            if stats is not None:
                stats.steps += 1
            if how is None:
                if stats is not None:
                    stats.skipped += 1
                continue
            out = ops.block(qs[r], ks[s], vs[s], how == "causal", scale, state,
                            done, nblocks)
            done += 1
            if done == nblocks:
                result = out
            if stats is not None:
                stats.blocks += 1
        outs.append(result[0])
        lses.append(result[1])
    return outs, lses
