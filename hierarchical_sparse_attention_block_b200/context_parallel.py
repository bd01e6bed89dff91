"""Decode with the KV cache split across ranks along the sequence (context parallelism).

Rank r of G holds tokens [t0, t0 + n_loc) of every sequence, whole blocks of
the block size B (the last rank may end on a partial block).  One decode step
runs the path on the local slice and exchanges three small sets between the
ranks (include/hisa.h, "Decode with the context split across ranks"):

1. every rank's best top_m - 2 blocks (+ the forced first / own block it
   owns) -> all-gather -> the global top-m blocks (`hisa_topk_merge`);
2. every rank's best top_k tokens of those blocks -> all-gather -> the global
   top-k tokens;
3. every rank's attention over the selected tokens it holds, as (O, LSE) ->
   all-gather -> the log-sum-exp merge.

The selections are exact: both are the best entries under one total order
(score descending, index ascending), and the global best are among the union
of every rank's best.  Messages per query: top_m + top_k (score, id) pairs
and H (d + 1) values per rank.

`exchange(t)` must return the tensors of every rank stacked in rank order
(an all-gather); `all_gather_exchange` builds it over torch.distributed (NCCL
on GPUs).  `Phases` holds the per-rank work between the exchanges; every
method is a call into the CUDA library.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (HisaParams, hisa_block_candidates, hisa_lse_merge, hisa_remap_ids, hisa_token_topk,
               hisa_topk_merge, sparse_attn_fwd)


@dataclass(frozen=True)
class Shard:
    """Tokens [t0, t0 + n_loc) of every sequence of an n_kv_global-token context, on rank `rank` of `world`."""

    rank: int
    world: int
    n_kv_global: int
    block: int
    t0: int
    n_loc: int

    @staticmethod
    def even(n_kv_global: int, block: int, rank: int, world: int) -> "Shard":
        """Whole blocks split as evenly as possible, in rank order."""
        n_blk = -(-n_kv_global // block)
        b0, b1 = rank * n_blk // world, (rank + 1) * n_blk // world
        t0, t1 = b0 * block, min(b1 * block, n_kv_global)
        return Shard(rank, world, n_kv_global, block, t0, t1 - t0)

    @property
    def first_block(self) -> int:
        return self.t0 // self.block

    @property
    def n_blk(self) -> int:
        return -(-self.n_loc // self.block)


def local_params(p, shard: Shard):
    """The rank's problem: its n_loc tokens, one query (the newest token of the whole context)."""
    pl = HisaParams.from_buffer_copy(p)
    pl.n_kv = shard.n_loc
    pl.n_q = 1
    return pl


class Phases:
    """This rank's part of a step between the exchanges, on the CUDA library."""

    def __init__(self, stream=None):
        self.stream = stream

    def blocks(self, pl, shard: Shard, q_idx, block_keys, idx_weights=None):
        import torch

        b, m = pl.batch, pl.top_m
        scores = torch.empty((b, m), dtype=torch.float32, device=q_idx.device)
        ids = torch.empty((b, m), dtype=torch.int32, device=q_idx.device)
        hisa_block_candidates(pl, shard.n_kv_global, shard.first_block, q_idx, block_keys, scores, ids,
                              stream=self.stream, idx_weights=idx_weights)
        return scores, ids

    def merge(self, scores_all, ids_all, k):
        import torch

        _, rows, _ = scores_all.shape
        out_ids = torch.empty((rows, k), dtype=torch.int32, device=ids_all.device)
        out_scores = torch.empty((rows, k), dtype=torch.float32, device=ids_all.device)
        hisa_topk_merge(scores_all, ids_all, k, out_ids, out_scores, stream=self.stream)
        return out_ids, out_scores

    def tokens(self, pl, shard: Shard, q_idx, k_idx, block_idx, status=None, idx_weights=None):
        import torch

        b = pl.batch
        dev = q_idx.device
        local_blk = torch.empty((b, 1, pl.top_m), dtype=torch.int32, device=dev)
        hisa_remap_ids(block_idx, shard.first_block, shard.first_block + shard.n_blk, -shard.first_block,
                       out=local_blk, stream=self.stream)
        tok = torch.empty((b, 1, pl.top_k), dtype=torch.int32, device=dev)
        scores = torch.empty((b, 1, pl.top_k), dtype=torch.float32, device=dev)
        hisa_token_topk(pl, q_idx, k_idx, local_blk, tok, scores, status, stream=self.stream, idx_weights=idx_weights)
        hisa_remap_ids(tok, 0, shard.n_loc, shard.t0, stream=self.stream)  # local -> global ids, in place
        return scores.view(b, pl.top_k), tok.view(b, pl.top_k)

    def attention(self, pl, shard: Shard, q, k, v, token_idx, status=None):
        import torch

        b = pl.batch
        dev = q.device
        local_tok = torch.empty((b, 1, pl.top_k), dtype=torch.int32, device=dev)
        hisa_remap_ids(token_idx, shard.t0, shard.t0 + shard.n_loc, -shard.t0, out=local_tok, stream=self.stream)
        o = torch.empty((b, 1, pl.n_heads, pl.d_head), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((b, 1, pl.n_heads), dtype=torch.float32, device=dev)
        sparse_attn_fwd(pl, q, k, v, local_tok, o, lse, status, stream=self.stream)
        return o, lse

    def lse_merge(self, o_all, lse_all):
        import torch

        o = torch.empty(o_all.shape[1:], dtype=o_all.dtype, device=o_all.device)
        lse = torch.empty(lse_all.shape[1:], dtype=lse_all.dtype, device=lse_all.device)
        hisa_lse_merge(o_all, lse_all, o, lse, stream=self.stream)
        return o, lse


def decode_step(p, shard: Shard, q_idx, k_idx, block_keys, q, k, v, exchange, phases=None, status=None,
                idx_weights=None):
    """One decode step of the whole context, run by every rank on its slice.

    p: the global problem (n_kv = the whole context, n_q = 1).  q_idx, q: the
    new token's indexer query and attention queries (the same on every rank);
    k_idx, k, v, block_keys: this rank's slice of the caches and its pooled
    block keys.  Returns (block_idx [b][m], token_idx [b][k], o, lse) of the
    whole context, the same on every rank.  idx_weights: the indexer's head weights with a
    multi-head indexer (p.n_idx_heads > 0), the same on every rank.
    """
    ph = phases if phases is not None else Phases()
    pl = local_params(p, shard)
    cs, ci = ph.blocks(pl, shard, q_idx, block_keys, idx_weights)
    blk, _ = ph.merge(exchange(cs), exchange(ci), p.top_m)
    ts, ti = ph.tokens(pl, shard, q_idx, k_idx, blk, status, idx_weights)
    tok, _ = ph.merge(exchange(ts), exchange(ti), p.top_k)
    o_part, lse_part = ph.attention(pl, shard, q, k, v, tok, status)
    o, lse = ph.lse_merge(exchange(o_part), exchange(lse_part))
    return blk, tok, o, lse


def all_gather_exchange(group=None):
    """exchange(t) over torch.distributed: every rank's t stacked in rank order."""
    import torch
    import torch.distributed as dist

    def exchange(t):
        t = t.contiguous()
        world = dist.get_world_size(group)
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t, group=group)
        return torch.stack(parts)

    return exchange

