"""Star Attention across GPUs: the pages' own multi-host form.

(hotaipapers.com page, Phase 1 and Phase 2 paragraphs; the authors' replies on
communication: Phase 1 needs no exchange besides the anchor, Phase 2 one vector
and one scalar per host and query row.)

- The context's blocks are spread over the ranks in contiguous runs; rank 0 holds
  b_0. Rank 0 broadcasts b_0's K/V (the anchor) once per layer into every rank's
  own memory. Each rank runs Phase 1 on its own blocks: rank 0 directly (its
  context starts with b_0), the others with star_attn_phase1_anchored, which reads
  the received anchor where it lies: no copy of the anchor next to the blocks, no
  anchor rows computed.
- Phase 2: the query host (the last rank by default) broadcasts the query rows; every
  rank attends with its own context keys (and the query host also with its
  query-local cache) and returns an fp32 output and an LSE per row
  (star_attn_phase2_partial); they are gathered to the query host only and
  merged exactly there (star_attn_lse_merge).

The collectives go through torch.distributed (NCCL between GPUs); the compute is
this library's kernels. `backend` lets the host logic run with other compute (the
tests drive it with the CPU oracle over gloo).
"""
from __future__ import annotations

import math
from typing import Optional

import torch


class GpuBackend:
    """The library's kernels."""

    def __init__(self):
        from . import lse_merge, phase1, phase1_anchored, phase2_partial
        self._phase1, self._partial, self._merge = phase1, phase2_partial, lse_merge
        self._anchored = phase1_anchored

    def phase1(self, q, k, v, block_size):
        return self._phase1(q, k, v, block_size)

    def phase1_anchored(self, q, k, v, k_anchor, v_anchor, block_size):
        return self._anchored(q, k, v, k_anchor, v_anchor, block_size)

    def partial(self, q, block_size, k_ctx, v_ctx, k, v, k_cache, v_cache, cache_len):
        return self._partial(q, block_size, k_ctx=k_ctx, v_ctx=v_ctx, k=k, v=v, k_cache=k_cache,
                             v_cache=v_cache, cache_len=cache_len)

    def lse_merge(self, o_parts, lse_parts):
        return self._merge(o_parts, lse_parts)


class ShardedStarAttention:
    """One attention layer's share on this rank.

        att = ShardedStarAttention(b, Hq, Hkv, d, ctx_len, block_size, cache_capacity)
        t0, t1 = att.token_range()                 # the context tokens this rank holds
        o_ctx, lse = att.prefill(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1])   # Phase 1 rows
        o_q = att.query(q_q, k_q, v_q)             # merged output on the query rank
        o_t = att.decode(q_t, k_t, v_t)            # one decode step (repeat)
    """

    def __init__(self, batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
                 cache_capacity, query_rank: Optional[int] = None, group=None, backend=None,
                 device="cuda", dtype=torch.bfloat16):
        dist = torch.distributed
        self.dist = dist if dist.is_available() and dist.is_initialized() else None
        self.group = group
        self.world = self.dist.get_world_size(group) if self.dist else 1
        self.rank = self.dist.get_rank(group) if self.dist else 0
        self.query_rank = self.world - 1 if query_rank is None else query_rank
        self.b, self.hq, self.hkv, self.d = batch, num_q_heads, num_kv_heads, head_dim
        self.L, self.B = ctx_len, min(block_size, ctx_len)
        self.backend = backend or GpuBackend()
        self.device, self.dtype = device, dtype
        n = math.ceil(ctx_len / self.B)
        lo, hi = self.rank * n // self.world, (self.rank + 1) * n // self.world
        self.t0, self.t1 = min(lo * self.B, ctx_len), min(hi * self.B, ctx_len)
        self.k_ctx = self.v_ctx = None
        self.k_cache = self.v_cache = None
        if self.rank == self.query_rank:
            self.k_cache = torch.zeros((batch, cache_capacity, num_kv_heads, head_dim),
                                       dtype=dtype, device=device)
            self.v_cache = torch.zeros_like(self.k_cache)
        self.cache_len = 0

    def token_range(self):
        return self.t0, self.t1

    # ------------------------------------------------------------------ Phase 1
    def prefill(self, q, k, v):
        """q, k, v: this rank's context tokens [b, t1 - t0, heads, d]. Returns this
        rank's Phase-1 rows (o, lse), or (None, None) if it holds no block."""
        B = self.B
        anchor_k = torch.empty((self.b, B, self.hkv, self.d), dtype=self.dtype, device=self.device)
        anchor_v = torch.empty_like(anchor_k)
        if self.rank == 0:
            anchor_k.copy_(k[:, :B])
            anchor_v.copy_(v[:, :B])
        if self.dist and self.world > 1:
            src = self.dist.get_global_rank(self.group, 0) if self.group else 0
            self.dist.broadcast(anchor_k, src=src, group=self.group)
            self.dist.broadcast(anchor_v, src=src, group=self.group)
        if self.t1 == self.t0:
            return None, None
        self.k_ctx, self.v_ctx = k, v
        if self.t0 == 0:
            return self.backend.phase1(q, k, v, B)
        # Every block here is a block i > 0: it attends to the received anchor and
        # causally to itself.
        return self.backend.phase1_anchored(q, k, v, anchor_k, anchor_v, B)

    # ------------------------------------------------------------------ Phase 2
    def _partial(self, q, k, v, cache_len):
        on_host = self.rank == self.query_rank
        if self.k_ctx is None and not on_host:
            rows = q.shape[1]
            o = torch.zeros((self.b, rows, self.hq, self.d), dtype=torch.float32 if q.is_cuda
                            else q.dtype, device=q.device)
            return o, torch.full((self.b, self.hq, rows), float("-inf"), dtype=o.dtype,
                                 device=q.device)
        return self.backend.partial(q, self.B, self.k_ctx, self.v_ctx,
                                    k if on_host else None, v if on_host else None,
                                    self.k_cache if on_host else None,
                                    self.v_cache if on_host else None, cache_len)

    def _combine(self, o, lse):
        """Gather every rank's (o, lse) to the query rank (one vector and one scalar
        per row and head from each host) and merge them there."""
        on_host = self.rank == self.query_rank
        if self.dist and self.world > 1:
            dst = self.dist.get_global_rank(self.group, self.query_rank) if self.group else self.query_rank
            os_ = [torch.empty_like(o) for _ in range(self.world)] if on_host else None
            ls = [torch.empty_like(lse) for _ in range(self.world)] if on_host else None
            self.dist.gather(o.contiguous(), os_, dst=dst, group=self.group)
            self.dist.gather(lse.contiguous(), ls, dst=dst, group=self.group)
        else:
            os_, ls = [o], [lse]
        if not on_host:
            return None, None
        return self.backend.lse_merge(torch.stack(os_), torch.stack(ls))

    def _broadcast_query(self, q):
        if self.dist and self.world > 1:
            q = q.contiguous()
            src = self.dist.get_global_rank(self.group, self.query_rank) if self.group else self.query_rank
            self.dist.broadcast(q, src=src, group=self.group)
        return q

    def query(self, q, k, v):
        """The query tokens: q [b, Lq, Hq, d] (taken from the query rank), k, v
        [b, Lq, Hkv, d] (used on the query rank). Returns (o, lse) on the query rank."""
        q = self._broadcast_query(q)
        o, lse = self._partial(q, k, v, 0)
        out = self._combine(o, lse)
        if self.rank == self.query_rank:
            self.cache_len = q.shape[1]
        return out

    def decode(self, q, k, v):
        """One decode step: q [b, 1, Hq, d], k, v [b, 1, Hkv, d]."""
        q = self._broadcast_query(q)
        o, lse = self._partial(q, k, v, self.cache_len)
        out = self._combine(o, lse)
        if self.rank == self.query_rank:
            self.cache_len += 1
        return out
