"""Vocabulary-parallel LM head over several GPUs, one process per GPU.

Each rank holds one contiguous shard of the head's rows, runs the fused
GEMM + online log-sum-exp + top-16 kernel over it (records with global
vocabulary indices), and the ranks' records are all-gathered in rank order
and merged by the same kernel that merges a single GPU's records.  The one
exchange is the records: M x P x 144 bytes per rank (P = 148 records per row
on a B200), small next to the shard of W each rank streams.

This module is orchestration only: every step of the arithmetic runs in the
library's kernels (dflash_lmhead_topk_partial, dflash_lmhead_topk_merge); the
collective is torch.distributed's all-gather (NCCL between GPUs).
"""
from __future__ import annotations

import torch

from . import _binding as _b

UNIT = 16   # shard boundaries fall on 16-row units (TMA-aligned rows of W)


def vocab_shard(V: int, world: int, rank: int, unit: int = UNIT):
    """Rows [v0, v1) of a V-row head owned by `rank`: contiguous, the world's
    shards cover [0, V) exactly once, balanced at `unit`-row granularity."""
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    units = (V + unit - 1) // unit
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(V, u0 * unit), min(V, u1 * unit)


def empty_records(M: int, P: int, device) -> torch.Tensor:
    """[M, P, 36] records that the merge ignores (max -inf, sum 0, values
    -inf, indices 0x7fffffff)."""
    r = torch.zeros((M, P, _b.RECORD_WORDS), dtype=torch.float32, device=device)
    r[:, :, 0] = float("-inf")
    r[:, :, 4:20] = float("-inf")
    r.view(torch.int32)[:, :, 20:36] = 0x7FFFFFFF
    return r


class VocabParallelLMHead:
    """LM head + log-softmax + top-16 over a vocabulary sharded across ranks.

    W_shard: this rank's rows [v0, v1) of the [V, d] head (bf16, on this
    rank's GPU); v0: the shard's first row.  Calling it with this rank's
    hidden states H [M, d] (the same H on every rank) returns the full
    vocabulary's (topk_logp, topk_idx, lse) on every rank.

    `partial_fn(H, W_shard, v0) -> records [M, P, 36]` and
    `merge_fn(records [world, M, P, 36]) -> (logp, idx, lse)` default to the
    library's kernels; they are parameters so the rank logic can be exercised
    on CPU process groups."""

    def __init__(self, W_shard, v0: int, group=None, partial_fn=None, merge_fn=None):
        self.W, self.v0, self.group = W_shard, int(v0), group
        self.partial_fn = partial_fn or (lambda H, W, off: _b.dflash_lmhead_topk_partial(H, W, v_offset=off))
        self.merge_fn = merge_fn or _b.dflash_lmhead_topk_merge

    def __call__(self, H):
        import torch.distributed as dist
        world = dist.get_world_size(self.group)
        local = self.partial_fn(H, self.W, self.v0)
        M, P_local, _ = local.shape
        # every rank gathers the same record count: pad to the largest
        p = torch.tensor([P_local], dtype=torch.int64, device=local.device)
        dist.all_reduce(p, op=dist.ReduceOp.MAX, group=self.group)
        P = int(p.item())
        if P_local < P:
            padded = empty_records(M, P, local.device)
            padded[:, :P_local] = local
            local = padded
        parts = [torch.empty_like(local) for _ in range(world)]
        dist.all_gather(parts, local.contiguous(), group=self.group)
        return self.merge_fn(torch.stack(parts))
