"""Plain float64 CPU oracle for Star Attention's two-phase attention (test infrastructure).

Only tests, the smoke check and the benchmark's CPU-baseline leg may call this
module. It is deliberately slow and direct: numpy matrix products and an
explicit visibility mask, no tiling, no online softmax, no fusion.

Notation (the Star Attention pages' terms): the context of L tokens is cut into
n = ceil(L / B) blocks b_0 .. b_{n-1} of B tokens (the last one may be short);
b_0 is the anchor block. Heads follow grouped-query attention: q-head h reads
kv-head h // (Hq / Hkv). Scores are s(t, j) = scale * <q_t, k_j>; the
log-sum-exp (LSE) of a row is ln sum_j exp(s(t, j)) over its visible keys.

Readings where the pages are silent (each is listed in the design notes):
  * softmax scale 1/sqrt(d) unless the caller gives one;
  * the Phase-2 "scalar" each block returns is the natural-log LSE of its
    scaled logits, and the "vector" is its softmax-normalised output;
  * the anchor's keys and values are b_0's own (inputs are already projected,
    so anchor tokens carry b_0's positions); anchor rows are not outputs;
  * query token j sees the whole context and query tokens 0..j; a decoded token
    sees everything cached before it and itself;
  * contiguous GQA grouping h -> h // (Hq / Hkv).
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

F64 = np.float64
_ROW_CHUNK = 1024


def default_scale(head_dim: int) -> float:
    """Softmax scale when the caller passes none: 1/sqrt(d), the standard
    scaled-dot-product choice (the pages do not state one)."""
    return 1.0 / math.sqrt(head_dim)


def kv_head_of(h: int, num_q_heads: int, num_kv_heads: int) -> int:
    """GQA mapping: q-head h reads kv-head h // G with G = Hq / Hkv."""
    return h // (num_q_heads // num_kv_heads)


def block_plan(ctx_len: int, block_size: int) -> List[Tuple[int, int]]:
    """Context blocking (hotaipapers.com page, Phase 1 paragraph: the context is
    split into blocks). Returns [start, end) of b_0 .. b_{n-1}, n = ceil(L/B);
    the last block may be shorter than B."""
    n = -(-ctx_len // block_size)
    return [(i * block_size, min(ctx_len, (i + 1) * block_size)) for i in range(n)]


def phase1_visible(t, j, block_size: int):
    """Phase-1 visibility of key position j to query position t (broadcasts).

    Causal attention over [anchor = b_0 ; b_i] for the block b_i holding t
    (hotaipapers.com page, Phase 1 paragraph: a copy of the first block is put
    in front of every other block; rebuttal to EMsM, "Size of Anchor Block":
    the anchor is as large as a block and Phase 1 is causal). So j is visible
    when j <= t and j lies either in the anchor b_0 or in t's own block. For
    t in b_0 both conditions name the same block: plain causal attention.
    """
    t = np.asarray(t)
    j = np.asarray(j)
    return (j <= t) & ((j < block_size) | (j // block_size == t // block_size))


def attend(q, k, v, scale: float, allowed=None) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of rows q [R, d] over keys k, v [N, d], in float64.

    This is one host's local attention in Phase 2 (hotaipapers.com page, Phase 2
    paragraph): it returns the output vector o [R, d] and the scalar
    lse [R] = ln sum_j exp(s_j) over the keys where `allowed` [R, N] is true.
    A row that sees no key returns o = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    s = scale * (q @ k.T)
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe[:, None])
    l = e.sum(axis=1)
    empty = l == 0
    l_safe = np.where(empty, 1.0, l)
    o = (e @ v) / l_safe[:, None]
    lse = m_safe + np.log(l_safe)
    o[empty] = 0.0
    lse[empty] = -np.inf
    return o, lse


def lse_merge(o_parts, lse_parts) -> Tuple[np.ndarray, np.ndarray]:
    """Query-host aggregation of per-block partials (hotaipapers.com page,
    Phase 2 paragraph: each host sends one vector and one scalar and the query
    host combines them into global attention).

    With partials (o_s, lse_s), s = 1..S, over disjoint key sets, the exact
    attention over their union is
        lse = M + ln sum_s exp(lse_s - M),   M = max_s lse_s
        o   = sum_s exp(lse_s - lse) * o_s
    Partials with lse_s = -inf (no visible key) weigh nothing.
    o_parts: [S, ..., d], lse_parts: [S, ...].
    """
    o_parts = np.asarray(o_parts, dtype=F64)
    lse_parts = np.asarray(lse_parts, dtype=F64)
    M = lse_parts.max(axis=0)
    M_safe = np.where(np.isfinite(M), M, 0.0)
    w = np.exp(lse_parts - M_safe)
    W = w.sum(axis=0)
    empty = W == 0
    W_safe = np.where(empty, 1.0, W)
    lse = M_safe + np.log(W_safe)
    o = (w[..., None] * o_parts).sum(axis=0) / W_safe[..., None]
    lse = np.where(empty, -np.inf, lse)
    o = np.where(empty[..., None], 0.0, o)
    return o, lse


def phase1_head(q, k, v, block_size: int, scale: float, rows: Sequence[int] = None):
    """Phase 1 for one (batch, q-head): q [L, d] and its kv-head's k, v [L, d].

    Each block b_i runs causal attention over [anchor = b_0 ; b_i] and keeps
    only its own rows (hotaipapers.com page, Phase 1 paragraph). For the rows of
    b_i the candidate keys are b_0 and b_i (every key `phase1_visible` can
    allow); the mask then applies the definition exactly.
    Returns o [R, d], lse [R] for `rows` (default: all L rows, in order).
    """
    L, d = q.shape[0], q.shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    o_out = np.zeros((len(rows), d), dtype=F64)
    lse_out = np.zeros(len(rows), dtype=F64)
    for start, end in block_plan(L, block_size):
        sel = np.nonzero((rows >= start) & (rows < end))[0]
        if sel.size == 0:
            continue
        if start == 0:
            cand = np.arange(0, end)
        else:
            cand = np.concatenate([np.arange(0, block_size), np.arange(start, end)])
        kc = np.asarray(k[cand], dtype=F64)
        vc = np.asarray(v[cand], dtype=F64)
        for c0 in range(0, sel.size, _ROW_CHUNK):
            idx = sel[c0:c0 + _ROW_CHUNK]
            t = rows[idx]
            allowed = phase1_visible(t[:, None], cand[None, :], block_size)
            o, lse = attend(q[t], kc, vc, scale, allowed)
            o_out[idx] = o
            lse_out[idx] = lse
    return o_out, lse_out


def phase1(q, k, v, block_size: int, scale: float = None):
    """Phase 1 over whole tensors: q [b, L, Hq, d], k, v [b, L, Hkv, d].
    Returns o [b, L, Hq, d] and lse [b, Hq, L] in float64."""
    b, L, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = default_scale(d) if scale is None else scale
    o = np.zeros((b, L, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, L), dtype=F64)
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            oh, lh = phase1_head(q[bi, :, h], k[bi, :, g], v[bi, :, g], block_size, scale)
            o[bi, :, h] = oh
            lse[bi, h] = lh
    return o, lse


def phase1_varlen(q, k, v, cu_seqlens: Sequence[int], block_size: int, scale: float = None):
    """Phase 1 over a varlen batch: sequences packed along the token axis,
    q [total, Hq, d], k, v [total, Hkv, d], sequence i = tokens
    [cu_seqlens[i], cu_seqlens[i+1]). Each sequence is its own context (its own
    blocks and anchor), so this is Phase 1 applied to each slice on its own.
    Returns o [total, Hq, d] and lse [Hq, total] in float64."""
    total, Hq, d = q.shape
    o = np.zeros((total, Hq, d), dtype=F64)
    lse = np.zeros((Hq, total), dtype=F64)
    for a, e in zip(cu_seqlens[:-1], cu_seqlens[1:]):
        if e == a:
            continue
        oi, li = phase1(q[None, a:e], k[None, a:e], v[None, a:e], block_size, scale)
        o[a:e] = oi[0]
        lse[:, a:e] = li[0]
    return o, lse


def phase2_query_head(q, k_ctx, v_ctx, k_qry, v_qry, scale: float):
    """Phase-2 query tokens by the definition: sequence-global attention
    (abstract: query and response tokens attend to all prior cached tokens).
    Query token j sees all L context keys and query keys 0..j.
    q [Lq, d]; k_ctx, v_ctx [L, d]; k_qry, v_qry [Lq, d]. Returns o [Lq, d], lse [Lq].
    """
    L = k_ctx.shape[0]
    Lq = q.shape[0]
    keys = np.concatenate([np.asarray(k_ctx, F64), np.asarray(k_qry, F64)])
    vals = np.concatenate([np.asarray(v_ctx, F64), np.asarray(v_qry, F64)])
    c = np.arange(L + Lq)[None, :]
    j = np.arange(Lq)[:, None]
    allowed = (c < L) | (c - L <= j)
    return attend(q, keys, vals, scale, allowed)


def phase2_query_head_blockwise(q, k_ctx, v_ctx, k_qry, v_qry, block_size: int, scale: float):
    """Phase-2 query tokens the way the pages compute them (hotaipapers.com page,
    Phase 2 paragraph): every context block b_i returns (o_i, lse_i) of the query
    over its own keys, the query host adds its own causal partial over the query
    tokens' KV, and the partials are merged with `lse_merge`."""
    L = k_ctx.shape[0]
    Lq = q.shape[0]
    o_parts, lse_parts = [], []
    for start, end in block_plan(L, block_size):
        o, lse = attend(q, k_ctx[start:end], v_ctx[start:end], scale)
        o_parts.append(o)
        lse_parts.append(lse)
    causal = np.arange(Lq)[None, :] <= np.arange(Lq)[:, None]
    o, lse = attend(q, k_qry, v_qry, scale, causal)
    o_parts.append(o)
    lse_parts.append(lse)
    return lse_merge(np.stack(o_parts), np.stack(lse_parts))


def phase2_query(q_qry, k_qry, v_qry, k_ctx, v_ctx, scale: float = None):
    """Phase-2 query over whole tensors: q_qry [b, Lq, Hq, d], k_qry, v_qry
    [b, Lq, Hkv, d], k_ctx, v_ctx [b, L, Hkv, d]. Returns o [b, Lq, Hq, d],
    lse [b, Hq, Lq]. The query tokens' KV become cache rows 0..Lq-1."""
    b, Lq, Hq, d = q_qry.shape
    Hkv = k_ctx.shape[2]
    scale = default_scale(d) if scale is None else scale
    o = np.zeros((b, Lq, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, Lq), dtype=F64)
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            oh, lh = phase2_query_head(q_qry[bi, :, h], k_ctx[bi, :, g], v_ctx[bi, :, g],
                                       k_qry[bi, :, g], v_qry[bi, :, g], scale)
            o[bi, :, h] = oh
            lse[bi, h] = lh
    return o, lse


def phase2_decode_head(q, k_ctx, v_ctx, k_cache, v_cache, k_new, v_new, scale: float):
    """One decode step for one (batch, q-head) (hotaipapers.com page, Phase 2
    paragraph: the query host appends the new token's KV to its cache, and the
    token attends globally). The token sees every context key, the cached query
    and earlier decode keys (k_cache [n, d]) and its own new key.
    q, k_new, v_new [d]. Returns o [d], lse (a float)."""
    keys = np.concatenate([np.asarray(k_ctx, F64), np.asarray(k_cache, F64),
                           np.asarray(k_new, F64)[None, :]])
    vals = np.concatenate([np.asarray(v_ctx, F64), np.asarray(v_cache, F64),
                           np.asarray(v_new, F64)[None, :]])
    o, lse = attend(np.asarray(q, F64)[None, :], keys, vals, scale)
    return o[0], lse[0]


def phase2_decode(q_t, k_t, v_t, k_ctx, v_ctx, k_cache, v_cache, cache_len: int,
                  scale: float = None):
    """One decode step over whole tensors: q_t [b, 1, Hq, d], k_t, v_t
    [b, 1, Hkv, d], caches [b, cap, Hkv, d] holding `cache_len` valid rows.
    Returns o [b, 1, Hq, d], lse [b, Hq, 1] and copies of the caches with the new
    token's KV appended at row cache_len."""
    b, _, Hq, d = q_t.shape
    Hkv = k_ctx.shape[2]
    scale = default_scale(d) if scale is None else scale
    o = np.zeros((b, 1, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, 1), dtype=F64)
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            oh, lh = phase2_decode_head(q_t[bi, 0, h], k_ctx[bi, :, g], v_ctx[bi, :, g],
                                        k_cache[bi, :cache_len, g], v_cache[bi, :cache_len, g],
                                        k_t[bi, 0, g], v_t[bi, 0, g], scale)
            o[bi, 0, h] = oh
            lse[bi, h, 0] = lh
    k_cache_new = np.array(k_cache, dtype=F64, copy=True)
    v_cache_new = np.array(v_cache, dtype=F64, copy=True)
    k_cache_new[:, cache_len] = np.asarray(k_t, F64)[:, 0]
    v_cache_new[:, cache_len] = np.asarray(v_t, F64)[:, 0]
    return o, lse, k_cache_new, v_cache_new


def phase2_query_varlen(q_qry, k_qry, v_qry, k_ctx, v_ctx, cu_ctx: Sequence[int],
                        cu_q: Sequence[int], scale: float = None):
    """Phase-2 query tokens over a varlen batch: sequence i has context tokens
    [cu_ctx[i], cu_ctx[i+1]) of k_ctx, v_ctx [total_ctx, Hkv, d] and query tokens
    [cu_q[i], cu_q[i+1]) of q_qry [total_q, Hq, d], k_qry, v_qry [total_q, Hkv, d];
    each sequence is the batch-1 query pass of its own slices.
    Returns o [total_q, Hq, d] and lse [Hq, total_q]."""
    total_q, Hq, d = q_qry.shape
    o = np.zeros((total_q, Hq, d), dtype=F64)
    lse = np.zeros((Hq, total_q), dtype=F64)
    for i in range(len(cu_q) - 1):
        a, e = cu_q[i], cu_q[i + 1]
        c0, c1 = cu_ctx[i], cu_ctx[i + 1]
        if e == a:
            continue
        oi, li = phase2_query(q_qry[None, a:e], k_qry[None, a:e], v_qry[None, a:e],
                              k_ctx[None, c0:c1], v_ctx[None, c0:c1], scale)
        o[a:e] = oi[0]
        lse[:, a:e] = li[0]
    return o, lse


def phase2_decode_varlen(q_t, k_t, v_t, k_ctx, v_ctx, cu_ctx: Sequence[int], k_cache, v_cache,
                         cache_lens: Sequence[int], scale: float = None):
    """One decode step over a varlen batch: sequence i has the context tokens
    [cu_ctx[i], cu_ctx[i+1]) of the packed k_ctx, v_ctx [total, Hkv, d] and
    cache_lens[i] cached rows of k_cache, v_cache [b, cap, Hkv, d]; q_t [b, 1, Hq, d],
    k_t, v_t [b, 1, Hkv, d]. Each sequence is the decode step of its own slice.
    Returns o [b, 1, Hq, d], lse [b, Hq, 1] and the caches with every new row appended."""
    b, _, Hq, d = q_t.shape
    o = np.zeros((b, 1, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, 1), dtype=F64)
    k_new = np.array(k_cache, dtype=F64, copy=True)
    v_new = np.array(v_cache, dtype=F64, copy=True)
    for i in range(b):
        a, e = cu_ctx[i], cu_ctx[i + 1]
        oi, li, ki, vi = phase2_decode(q_t[i:i + 1], k_t[i:i + 1], v_t[i:i + 1], k_ctx[None, a:e],
                                       v_ctx[None, a:e], k_cache[i:i + 1], v_cache[i:i + 1],
                                       cache_lens[i], scale)
        o[i], lse[i], k_new[i], v_new[i] = oi[0], li[0], ki[0], vi[0]
    return o, lse, k_new, v_new


def rope(x, positions: Sequence[int], inv_freq: Sequence[float]):
    """Rotary position embedding in float64, rotate-half pairs: for x [..., L, H, d]
    and token positions [L], the pair (x[f], x[f + d/2]) of a token at position p
    is rotated by the angle p * inv_freq[f]."""
    x = np.asarray(x, F64)
    h = x.shape[-1] // 2
    ang = np.asarray(positions, F64)[:, None] * np.asarray(inv_freq, F64)[None, :]  # [L, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def phase1_rope_head(q_raw, k_raw, v, block_size: int, scale: float, inv_freq,
                     anchor_positions: str = "original"):
    """Phase 1 for one head with RoPE applied inside each block's local attention
    (rebuttal to x5MA, "Anchor Block Content and Position"). q_raw, k_raw [L, d] are
    the un-rotated projections, v [L, d]. Block tokens keep their own positions;
    the anchor (b_0's tokens) gets position j ("original") or (i-1)B + j
    ("adjacent": right before block i) in block i's local context.
    Returns o [L, d], lse [L]."""
    L, d = q_raw.shape
    B = block_size
    o = np.zeros((L, d), dtype=F64)
    lse = np.zeros(L, dtype=F64)
    rot = lambda x, pos: rope(np.asarray(x, F64)[:, None, :], pos, inv_freq)[:, 0]
    for start, end in block_plan(L, B):
        i = start // B
        own = np.arange(start, end)
        q = rot(q_raw[start:end], own)
        k_own = rot(k_raw[start:end], own)
        causal = own[None, :] <= own[:, None]
        if i == 0:
            keys, vals, allowed = k_own, np.asarray(v[start:end], F64), causal
        else:
            apos = np.arange(B) if anchor_positions == "original" else (i - 1) * B + np.arange(B)
            keys = np.concatenate([rot(k_raw[:B], apos), k_own])
            vals = np.concatenate([np.asarray(v[:B], F64), np.asarray(v[start:end], F64)])
            allowed = np.concatenate([np.ones((end - start, B), dtype=bool), causal], axis=1)
        o[start:end], lse[start:end] = attend(q, keys, vals, scale, allowed)
    return o, lse


def phase1_rope(q_raw, k_raw, v, block_size: int, inv_freq, anchor_positions: str = "original",
                scale: float = None):
    """phase1_rope_head over whole tensors: q_raw [b, L, Hq, d], k_raw, v [b, L, Hkv, d].
    Returns o [b, L, Hq, d] and lse [b, Hq, L]."""
    b, L, Hq, d = q_raw.shape
    Hkv = k_raw.shape[2]
    scale = default_scale(d) if scale is None else scale
    o = np.zeros((b, L, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, L), dtype=F64)
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            o[bi, :, h], lse[bi, h] = phase1_rope_head(q_raw[bi, :, h], k_raw[bi, :, g], v[bi, :, g],
                                                       block_size, scale, inv_freq, anchor_positions)
    return o, lse


def model_forward(x_ctx, x_qry, x_dec: Sequence, w_qkv: Sequence, w_o: Sequence, Hq: int, Hkv: int,
                  d: int, block_size: int, inv_freq, anchor_positions: str = "original"):
    """A stack of attention layers driven the Star Attention way, in float64: per
    layer, q|k|v = x W_qkv, RoPE at the tokens' positions (context 0..L-1, query
    L.., decode after them), Phase 1 over the context (phase1_rope: the anchor
    positions as chosen), Phase 2 for the query tokens and then each decode token
    (every layer keeps its rotated context K/V and its query-local cache), and
    x += o W_o. x_ctx [b, L, hidden], x_qry [b, Lq, hidden], x_dec: list of
    [b, 1, hidden]. Returns the hidden states after the last layer for the context,
    the query and every decode token."""
    b, L, _ = x_ctx.shape
    Lq = x_qry.shape[1]
    T = len(x_dec)
    qd, kd = Hq * d, Hkv * d

    def split(h, n):
        h = np.asarray(h, F64)
        return (h[..., :qd].reshape(b, n, Hq, d), h[..., qd:qd + kd].reshape(b, n, Hkv, d),
                h[..., qd + kd:].reshape(b, n, Hkv, d))

    xs = [np.asarray(x_ctx, F64), np.asarray(x_qry, F64)] + [np.asarray(t, F64) for t in x_dec]
    for li in range(len(w_qkv)):
        W, Wo = np.asarray(w_qkv[li], F64), np.asarray(w_o[li], F64)
        q, k, v = split(xs[0] @ W, L)
        o, _ = phase1_rope(q, k, v, block_size, inv_freq, anchor_positions)
        k_ctx = rope(k, np.arange(L), inv_freq)
        outs = [o]
        qq, kq, vq = split(xs[1] @ W, Lq)
        pos_q = L + np.arange(Lq)
        qq, kq = rope(qq, pos_q, inv_freq), rope(kq, pos_q, inv_freq)
        oq, _ = phase2_query(qq, kq, vq, k_ctx, v)
        outs.append(oq)
        cap = Lq + T
        kc = np.zeros((b, cap, Hkv, d))
        vc = np.zeros((b, cap, Hkv, d))
        kc[:, :Lq], vc[:, :Lq] = kq, vq
        for t in range(T):
            qt, kt, vt = split(xs[2 + t] @ W, 1)
            pos_t = [L + Lq + t]
            qt, kt = rope(qt, pos_t, inv_freq), rope(kt, pos_t, inv_freq)
            ot, _, kc, vc = phase2_decode(qt, kt, vt, k_ctx, v, kc, vc, Lq + t)
            outs.append(ot)
        xs = [x + oo.reshape(x.shape[0], x.shape[1], qd) @ Wo for x, oo in zip(xs, outs)]
    return xs[0], xs[1], xs[2:]


def phase2_partial(q, k_ctx, v_ctx, k_new, v_new, k_cache, v_cache, cache_len: int,
                   scale: float = None):
    """One host's share of Phase 2 (hotaipapers.com page, Phase 2 paragraph: each host
    attends with its own keys and returns one vector and one scalar per query row).
    Rows of q [b, rows, Hq, d] attend to this host's context keys k_ctx, v_ctx
    [b, L, Hkv, d] (all visible; None: no context) and, on the query host, to its
    query-local cache k_cache, v_cache [b, cap, Hkv, d] (None elsewhere): one row is a
    decode step whose k_new, v_new go to row cache_len and which sees rows
    0..cache_len; several rows are the query tokens, written to rows [0, rows), row j
    seeing rows 0..j. Returns o [b, rows, Hq, d], lse [b, Hq, rows] and the updated
    caches (None without a cache)."""
    q = np.asarray(q, F64)
    b, rows, Hq, d = q.shape
    Hkv = (k_ctx if k_ctx is not None else k_cache).shape[2]
    scale = default_scale(d) if scale is None else scale
    kc = vc = None
    if k_cache is not None:
        kc = np.array(k_cache, dtype=F64, copy=True)
        vc = np.array(v_cache, dtype=F64, copy=True)
        start = cache_len if rows == 1 else 0
        kc[:, start:start + rows] = np.asarray(k_new, F64)
        vc[:, start:start + rows] = np.asarray(v_new, F64)
    o = np.zeros((b, rows, Hq, d), dtype=F64)
    lse = np.zeros((b, Hq, rows), dtype=F64)
    for bi in range(b):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            keys, vals, masks = [], [], []
            if k_ctx is not None:
                n = k_ctx.shape[1]
                keys.append(np.asarray(k_ctx[bi, :, g], F64))
                vals.append(np.asarray(v_ctx[bi, :, g], F64))
                masks.append(np.ones((rows, n), dtype=bool))
            if kc is not None:
                last = np.full(rows, cache_len) if rows == 1 else np.arange(rows)
                n = int(last.max()) + 1
                keys.append(kc[bi, :n, g])
                vals.append(vc[bi, :n, g])
                masks.append(np.arange(n)[None, :] <= last[:, None])
            o[bi, :, h], lse[bi, h] = attend(q[bi, :, h], np.concatenate(keys),
                                             np.concatenate(vals), scale,
                                             np.concatenate(masks, axis=1))
    return o, lse, kc, vc
