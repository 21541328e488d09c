"""The QUOKA prefill-chunk step with the prior keys split over ranks.

Context parallelism for caches too long for one GPU: rank r of N holds a
contiguous shard of the T prior keys (and values) of every (batch, KV head),
shard r before shard r + 1, plus the whole chunk (Q, Kc, Vc). Every step is
a call of libquoka.so; torch.distributed carries the two exchanges:

  1. steps (a)-(e) on the shard (quoka_select with the global BSA) give the
     shard's top-min(BSA, T_r) keys; quoka_shard_candidate_scores pads them,
     with their scores, to C = min(BSA, max_r T_r);
  2. all-gather of the candidate scores (N, b, nkv, C), quoka_shard_interleave
     to rank-major rows, quoka_topk with BSA_eff = min(BSA, T_total);
  3. quoka_shard_take: this rank's share of the selection, as key indices of
     its shard;
  4. quoka_sparse_gqa_attn over that share (rank 0 also over the chunk's own
     keys; the other ranks pass the no-chunk option), with the log-sum-exp;
  5. all-gather of (O, lse), quoka_combine_partials.

The selection equals the one-device selection: a key of the global top-BSA
is among its own shard's top-BSA, and the concatenation keeps the global key
order, so ties at the BSA-th score still go to the lower key index. Steps
(a)-(c) depend on the chunk only and are repeated on every rank.

The steps are also exposed one by one (local_candidates, select_share,
partial_attention, combine) so that one process can run several shards in
turn; `ops` selects the implementation of the per-rank calls (the library,
by default).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import torch

from . import _lib


@dataclass(frozen=True)
class ShardPlan:
    """Sizes of the prior-key shards (rank order) and what follows from
    them."""
    T_shards: tuple
    BSA: int

    @property
    def N(self) -> int:
        return len(self.T_shards)

    @property
    def T_total(self) -> int:
        return int(sum(self.T_shards))

    @property
    def C(self) -> int:
        """Candidates per rank and row (the longest shard's min(BSA, T_r))."""
        return min(self.BSA, max(self.T_shards)) if self.T_shards else 0

    @property
    def BSA_eff(self) -> int:
        return min(self.BSA, self.T_total)

    def offset(self, rank: int) -> int:
        return int(sum(self.T_shards[:rank]))


class LibraryOps:
    """The per-rank calls, on libquoka.so."""

    def select(self, Q, K, NQ, BSA, dot_product=False):
        kv_idx, kv_count, _, s_agg = _lib.quoka_select(Q, K, NQ, BSA, want_s_agg=True, dot_product=dot_product)
        return kv_idx, kv_count, s_agg

    def candidates(self, s_agg, kv_idx, kv_count, C):
        return _lib.quoka_shard_candidate_scores(s_agg, kv_idx, kv_count, C)

    def interleave(self, gathered):
        return _lib.quoka_shard_interleave(gathered)

    def topk(self, scores, BSA):
        return _lib.quoka_topk(scores, BSA)

    def take(self, sel_pos, sel_count, cand_idx, rank):
        return _lib.quoka_shard_take(sel_pos, sel_count, cand_idx, rank)

    def attention(self, Q, K, V, kv_idx, kv_count, Kc, Vc, scale, with_chunk):
        return _lib.quoka_sparse_gqa_attn(Q, K, V, kv_idx, kv_count, Kc, Vc, scale, want_lse=True,
                                          no_chunk=not with_chunk)

    def combine(self, O_parts, lse_parts):
        return _lib.quoka_combine_partials(O_parts, lse_parts)


def local_candidates(plan: ShardPlan, Q, K_shard, NQ: int, *, dot_product=False, ops=None):
    """Steps (a)-(e) on this rank's shard; returns (scores, cand_idx), each
    (b, nkv, plan.C), padded with -inf / -1."""
    ops = ops or LibraryOps()
    kv_idx, kv_count, s_agg = ops.select(Q, K_shard, NQ, plan.BSA, dot_product)
    return ops.candidates(s_agg, kv_idx, kv_count, plan.C)


def select_share(plan: ShardPlan, all_scores, cand_idx, rank: int, *, ops=None):
    """The global top-BSA over the gathered candidate scores (N, b, nkv, C)
    and this rank's share of it: (kv_idx (b, nkv, C) int32 ascending key
    indices of the shard, kv_count (b, nkv))."""
    ops = ops or LibraryOps()
    rows = ops.interleave(all_scores)
    sel_pos, sel_count = ops.topk(rows, plan.BSA_eff)
    return ops.take(sel_pos, sel_count, cand_idx, rank)


def partial_attention(plan: ShardPlan, rank: int, Q, K_shard, V_shard, Kc, Vc, kv_idx, kv_count,
                      scale: Optional[float] = None, *, ops=None):
    """This rank's softmax attention over its share of the selection (rank 0
    also over the chunk's own keys): (O, lse)."""
    ops = ops or LibraryOps()
    if scale is None:
        scale = Q.shape[-1] ** -0.5
    return ops.attention(Q, K_shard, V_shard, kv_idx, kv_count, Kc, Vc, scale, rank == 0)


def combine(O_parts, lse_parts, *, ops=None):
    """Merge of the ranks' gathered (N, ...) partial outputs: (O, lse)."""
    ops = ops or LibraryOps()
    return ops.combine(O_parts, lse_parts)


def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    """(N, *t.shape) with rank r's tensor at index r."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    out = torch.empty((n,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    t = t.contiguous()
    if hasattr(dist, "all_gather_into_tensor") and t.is_cuda:
        dist.all_gather_into_tensor(out, t, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t, group=group)
    return out


def prefill_chunk_sharded(Q, K_shard, V_shard, Kc, Vc, NQ: int, BSA: int, T_shards: Sequence[int], *,
                          scale: Optional[float] = None, dot_product: bool = False, group=None,
                          ops=None, all_gather: Optional[Callable] = None):
    """Steps (a)-(g) with the prior keys split over the ranks of `group`
    (T_shards: every rank's shard length, rank order). Returns (O, lse,
    kv_idx, kv_count), the last two this rank's share of the selection."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    plan = ShardPlan(tuple(int(t) for t in T_shards), int(BSA))
    if plan.N != dist.get_world_size(group) or K_shard.shape[2] != plan.T_shards[rank]:
        raise ValueError("T_shards must list every rank's shard length, this rank's matching K_shard")
    gather = all_gather or (lambda t: _all_gather(t, group))
    scores, cand_idx = local_candidates(plan, Q, K_shard, NQ, dot_product=dot_product, ops=ops)
    kv_idx, kv_count = select_share(plan, gather(scores), cand_idx, rank, ops=ops)
    O_r, lse_r = partial_attention(plan, rank, Q, K_shard, V_shard, Kc, Vc, kv_idx, kv_count, scale, ops=ops)
    O, lse = combine(gather(O_r), gather(lse_r), ops=ops)
    return O, lse, kv_idx, kv_count
