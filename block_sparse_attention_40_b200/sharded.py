"""Context-sharded decode across ranks: host orchestration only.

A batch's contexts are split over R shards, rank r holding shard r (tokens
[t0_r, t0_r + capacity) of every sequence; see include/qsa.h, context-sharded decode).  One
decode step exchanges two things between the ranks:

1. every shard's top-k (score, global block) candidates, gathered in rank order so that every
   rank merges the same stack and reaches the same selection;
2. every shard's partial softmax (o, m, l), gathered in rank order and merged by log-sum-exp.

The arithmetic runs in the library's kernels (ShardDecoder.select / .attend,
merge_candidates, combine_partials); this module only moves their buffers with
torch.distributed (NCCL between GPUs; any backend works for the exchange itself).
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import binding as B


def _gather_stack(t: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' copies of t stacked in rank order: [world, *t.shape]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def exchange_candidates(cand_score: torch.Tensor, cand_idx: torch.Tensor,
                        cand_cnt: torch.Tensor, group=None):
    """This rank's shard candidates ([B, k], [B, k], [B]) -> every shard's, stacked in rank
    order ([R, B, k], [R, B, k], [R, B])."""
    return (_gather_stack(cand_score, group), _gather_stack(cand_idx, group),
            _gather_stack(cand_cnt, group))


def exchange_partials(part_o: torch.Tensor, part_m: torch.Tensor, part_l: torch.Tensor,
                      group=None):
    """This rank's partial softmax ([B, 24, 128], [B, 24], [B, 24]) -> every shard's, stacked
    in rank order."""
    return (_gather_stack(part_o, group), _gather_stack(part_m, group),
            _gather_stack(part_l, group))


def decode_step(shard: B.ShardDecoder, q, q_idx, w, glen: torch.Tensor, max_blocks: int,
                group=None):
    """One context-sharded decode step on this rank's shard (the new token already appended to
    the shard that holds it).  Returns the output [B, 24, 128] (identical on every rank) and
    the selection (idx, cnt)."""
    cs, ci, cc = shard.select(q_idx, w, glen)
    cs, ci, cc = exchange_candidates(cs, ci, cc, group)
    sel_idx, sel_cnt = B.merge_candidates(cs, ci, cc, shard.topk, max_blocks)
    po, pm, pl = shard.attend(q, glen, sel_idx, sel_cnt)
    po, pm, pl = exchange_partials(po, pm, pl, group)
    return B.combine_partials(po, pm, pl), sel_idx, sel_cnt


def decode_step_local(shards: Sequence[B.ShardDecoder], q, q_idx, w, glen: torch.Tensor,
                      max_blocks: int):
    """The same step with every shard on this process's device (no exchange): the candidates
    and partials are stacked in shard order directly."""
    cands = [s.select(q_idx, w, glen) for s in shards]
    cs = torch.stack([c[0] for c in cands])
    ci = torch.stack([c[1] for c in cands])
    cc = torch.stack([c[2] for c in cands])
    sel_idx, sel_cnt = B.merge_candidates(cs, ci, cc, shards[0].topk, max_blocks)
    parts = [s.attend(q, glen, sel_idx, sel_cnt) for s in shards]
    po = torch.stack([p[0] for p in parts])
    pm = torch.stack([p[1] for p in parts])
    pl = torch.stack([p[2] for p in parts])
    return B.combine_partials(po, pm, pl), sel_idx, sel_cnt


def shard_counts(lengths: Sequence[int], t0: int, capacity: int, lo: int, hi: int):
    """Tokens [lo, hi) of every sequence that fall in the shard [t0, t0 + capacity), as
    per-sequence counts for an append of the columns [max(lo, t0), min(hi, t0 + capacity))
    (sequence b has lengths[b] tokens in all)."""
    a, e = max(lo, t0), min(hi, t0 + capacity)
    return [max(0, min(e, L) - a) for L in lengths]
