"""Star Attention two-phase attention on B200 (sm_100a): Python binding.

A thin ctypes layer over the C-ABI library libstarattn.so (include/star_attn.h).
It only marshals arguments: it checks tensor dtypes/shapes, allocates outputs
with torch (device memory is PyTorch's job here), and passes raw pointers and
the current CUDA stream. Every step of the attention runs in the library's
CUDA kernels; there is no fallback of any kind. If the library is missing the
import of an entry point raises.

Entry points mirror the C names:
    phase1(q, k, v, block_size)                      -> (o, lse)
    phase2_query(q, k, v, k_ctx, v_ctx, k_cache, v_cache, block_size) -> (o, lse)
    phase2_decode(q, k, v, k_ctx, v_ctx, k_cache, v_cache, cache_len, block_size) -> (o, lse)
    lse_merge(o_parts, lse_parts)                    -> (o, lse)
and StarAttentionLayer bundles them with the caches and workspace of one layer.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# STAR_ATTN_LIBRARY may name another build of the same library (the debug build,
# libstarattn_debug.so next to this file); there is no other fallback.
LIB_PATH = os.environ.get("STAR_ATTN_LIBRARY") or os.path.join(_HERE, "libstarattn.so")

STAR_PHASE1, STAR_PHASE2_QUERY, STAR_PHASE2_DECODE, STAR_PHASE2_DECODE_FUSED = 1, 2, 3, 4
STATUS_NAMES = {0: "STAR_OK", 1: "STAR_ERR_INVALID_ARG", 2: "STAR_ERR_UNSUPPORTED",
                3: "STAR_ERR_WORKSPACE", 4: "STAR_ERR_CACHE_FULL", 5: "STAR_ERR_CUDA",
                6: "STAR_ERR_TIMEOUT"}

# Every symbol the header declares; tests check that the library exports them all.
EXPORTED = ["star_attn_workspace_bytes", "star_attn_phase1", "star_attn_phase1_varlen",
            "star_attn_phase1_anchored",
            "star_attn_rope", "star_attn_phase1_anchor_q",
            "star_attn_phase2_query",
            "star_attn_phase2_decode", "star_attn_phase2_decode_fused",
            "star_attn_phase2_decode_varlen", "star_attn_decode_varlen_workspace_bytes",
            "star_attn_phase2_query_varlen", "star_attn_query_varlen_workspace_bytes",
            "star_attn_phase2_partial",
            "star_attn_phase2_query_paged",
            "star_attn_phase2_decode_paged", "star_attn_phase2_decode_noalloc",
            "star_attn_lse_merge", "star_attn_simple_phase1",
            "star_attn_simple_phase2", "star_attn_get_device_status",
            "star_attn_selftest_wait_timeout", "star_attn_selftest_exp2", "star_attn_selftest_read",
            "star_attn_debug_build", "star_attn_debug_record", "star_attn_selftest_bounds",
            "star_attn_launch_count",
            "star_attn_status_string", "star_attn_version"]


class StarAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ctx_len", ctypes.c_int64), ("block_size", ctypes.c_int64),
                ("softmax_scale", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libstarattn.so (built in-tree by block_sparse_attention_phase_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m block_sparse_attention_phase_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    sig = {
        "star_attn_workspace_bytes": (SZ, [SP, I32, I64]),
        "star_attn_phase1": (I32, [SP, P, P, P, P, P, P]),
        "star_attn_phase1_varlen": (I32, [SP, ctypes.POINTER(I64), P, P, P, P, P, P]),
        "star_attn_phase1_anchored": (I32, [SP, P, P, P, P, P, P, P, P]),
        "star_attn_rope": (I32, [SP, ctypes.POINTER(ctypes.c_float), I64, P, P, P, P, P, P]),
        "star_attn_phase1_anchor_q": (I32, [SP, P, P, P, P, P, P, P]),
        "star_attn_phase2_query": (I32, [SP, P, P, P, I64, P, P, P, P, I64, P, P, P, SZ, P]),
        "star_attn_phase2_decode": (I32, [SP, P, P, P, P, P, P, P, I64, I64, P, P, P, SZ, P]),
        "star_attn_phase2_decode_fused": (I32, [SP, P, P, P, P, P, P, P, I64, I64, P, P, P, SZ,
                                                 P]),
        "star_attn_phase2_decode_varlen": (I32, [SP, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                                  P, P, P, P, P, P, P, I64, P, I32, I32, I32,
                                                  P, P, P, SZ, P]),
        "star_attn_decode_varlen_workspace_bytes": (SZ, [SP, ctypes.POINTER(I64)]),
        "star_attn_phase2_partial": (I32, [SP, P, P, P, I64, P, P, P, P, I64, I64, P, P, P, SZ,
                                           P]),
        "star_attn_phase2_query_varlen": (I32, [SP, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                                 P, P, P, P, P, P, P, I64, P, I32, I32, I32,
                                                 P, P, P, SZ, P]),
        "star_attn_query_varlen_workspace_bytes": (SZ, [SP, ctypes.POINTER(I64),
                                                        ctypes.POINTER(I64)]),
        "star_attn_phase2_query_paged": (I32, [SP, P, P, P, I64, P, P, P, P, I32, I32, P, I32,
                                                P, P, P, SZ, P]),
        "star_attn_phase2_decode_paged": (I32, [SP, P, P, P, P, P, P, P, I32, I32, P, I32, I64,
                                                 P, P, P, SZ, P]),
        "star_attn_phase2_decode_noalloc": (I32, [SP, P, P, P, P, P, P, P, I64, I64, P, P, P]),
        "star_attn_lse_merge": (I32, [P, P, I32, I32, I64, I32, I32, P, P, P]),
        "star_attn_simple_phase1": (I32, [SP, P, P, P, P, P, P]),
        "star_attn_simple_phase2": (I32, [SP, P, I64, P, P, P, P, I64, I64, I32, P, P, P]),
        "star_attn_get_device_status": (I32, [P]),
        "star_attn_selftest_wait_timeout": (I32, [ctypes.c_uint64, P]),
        "star_attn_selftest_exp2": (I32, [P, P, I64, P]),
        "star_attn_selftest_read": (I32, [P, SZ, P, I32, P]),
        "star_attn_debug_build": (I32, []),
        "star_attn_debug_record": (I32, [ctypes.POINTER(I64), P]),
        "star_attn_selftest_bounds": (I32, [P, I64, P]),
        "star_attn_launch_count": (ctypes.c_uint64, []),
        "star_attn_status_string": (ctypes.c_char_p, [I32]),
        "star_attn_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, what: str) -> None:
    if status != 0:
        raise StarAttnError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bf16(t: torch.Tensor, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor, got {tuple(t.shape)}")


def make_shape(batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
               softmax_scale: Optional[float] = None) -> Shape:
    return Shape(batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
                 0.0 if softmax_scale is None else float(softmax_scale))


def workspace_bytes(shape: Shape, phase: int, rows: int = 1) -> int:
    return int(lib().star_attn_workspace_bytes(ctypes.byref(shape), phase, rows))


def _ctx_shape(q, k, block_size, scale) -> Shape:
    b, L, hq, d = q.shape
    return make_shape(b, hq, k.shape[2], d, L, block_size, scale)


def phase1(q, k, v, block_size: int, scale: Optional[float] = None, o=None, lse=None,
           want_lse: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Anchor-prefixed blockwise-local causal attention over the context.
    q [b, L, Hq, d], k/v [b, L, Hkv, d] bf16 -> o [b, L, Hq, d] bf16, lse [b, Hq, L] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n, 4)
    shape = _ctx_shape(q, k, block_size, scale)
    b, L, hq, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((b, hq, L), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase1(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                  _ptr(lse), _stream()), "star_attn_phase1")
    return o, lse


def phase1_anchored(q, k, v, k_anchor, v_anchor, block_size: int, scale: Optional[float] = None,
                    o=None, lse=None, want_lse: bool = True):
    """One host's share of Phase 1: q [b, L, Hq, d], k/v [b, L, Hkv, d] are whole blocks
    b_i.. (i > 0) of a longer context; k_anchor/v_anchor [b, B, Hkv, d] are b_0's K/V.
    Every local block attends to the anchor and causally to itself. Returns (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_anchor, "k_anchor"), (v_anchor, "v_anchor")):
        _bf16(t, n, 4)
    if k_anchor.shape[1] != block_size or k_anchor.shape != v_anchor.shape:
        raise ValueError("the anchor holds block_size tokens of K and of V")
    shape = _ctx_shape(q, k, block_size, scale)
    b, L, hq, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((b, hq, L), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase1_anchored(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(k_anchor), _ptr(v_anchor), _ptr(o), _ptr(lse),
                                           _stream()), "star_attn_phase1_anchored")
    return o, lse


def rope_inv_freq(head_dim: int, base: float = 500000.0):
    """Plain RoPE frequencies base^(-2f/d), f < d/2, as float32 values."""
    import numpy as np
    f = np.arange(head_dim // 2, dtype=np.float64)
    return (base ** (-2.0 * f / head_dim)).astype(np.float32)


def rope(q, k, inv_freq, pos0: int = 0, block_size: int = 1, want_anchor: bool = False,
         inplace: bool = False):
    """RoPE on q [b, L, Hq, d] and k [b, L, Hkv, d] at positions pos0 + t. Returns
    (q_rot, k_rot, q_anchor or None); q_anchor is q rotated at the anchor-position
    variant's positions for blocks of block_size tokens."""
    _bf16(q, "q", 4)
    _bf16(k, "k", 4)
    b, L, hq, d = q.shape
    freqs = [float(x) for x in inv_freq]
    if len(freqs) != d // 2:
        raise ValueError("inv_freq needs head_dim / 2 entries")
    arr = (ctypes.c_float * len(freqs))(*freqs)
    shape = make_shape(b, hq, k.shape[2], d, L, block_size)
    qo = q if inplace else torch.empty_like(q)
    ko = k if inplace else torch.empty_like(k)
    qa = torch.empty_like(q) if want_anchor else None
    _check(lib().star_attn_rope(ctypes.byref(shape), arr, int(pos0), _ptr(q), _ptr(k), _ptr(qo),
                                _ptr(ko), _ptr(qa), _stream()), "star_attn_rope")
    return qo, ko, qa


def phase1_anchor_q(q, q_anchor, k, v, block_size: int, scale: Optional[float] = None,
                    o=None, lse=None, want_lse: bool = True):
    """Phase 1 whose anchor tiles are scored with q_anchor (anchor-position variant)."""
    for t, n in ((q, "q"), (q_anchor, "q_anchor"), (k, "k"), (v, "v")):
        _bf16(t, n, 4)
    shape = _ctx_shape(q, k, block_size, scale)
    b, L, hq, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((b, hq, L), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase1_anchor_q(ctypes.byref(shape), _ptr(q), _ptr(q_anchor), _ptr(k),
                                           _ptr(v), _ptr(o), _ptr(lse), _stream()),
           "star_attn_phase1_anchor_q")
    return o, lse


def _cu_array(cu_seqlens):
    vals = [int(x) for x in cu_seqlens]
    return (ctypes.c_int64 * len(vals))(*vals), vals


def phase1_varlen(q, k, v, cu_seqlens, block_size: int, scale: Optional[float] = None,
                  o=None, lse=None, want_lse: bool = True):
    """Phase 1 over sequences packed along tokens: q [total, Hq, d], k/v [total, Hkv, d],
    cu_seqlens = host offsets [n + 1] (list/array/CPU tensor). Returns (o [total, Hq, d],
    lse [Hq, total]); each sequence is computed as if alone."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n, 3)
    cu, vals = _cu_array(cu_seqlens)
    total, hq, d = q.shape
    shape = make_shape(len(vals) - 1, hq, k.shape[1], d, total, block_size, scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((hq, total), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase1_varlen(ctypes.byref(shape), cu, _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(o), _ptr(lse), _stream()), "star_attn_phase1_varlen")
    return o, lse


def _ws(shape: Shape, phase: int, rows: int, device, workspace):
    need = workspace_bytes(shape, phase, rows)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    return workspace


def phase2_query(q, k, v, k_ctx, v_ctx, k_cache, v_cache, block_size: int,
                 scale: Optional[float] = None, o=None, lse=None, workspace=None):
    """Query tokens: q [b, Lq, Hq, d], k/v [b, Lq, Hkv, d]; context KV [b, L, Hkv, d];
    caches [b, cap, Hkv, d] (rows 0..Lq-1 are written). Returns (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx"),
                 (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n, 4)
    b, lq, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    workspace = _ws(shape, STAR_PHASE2_QUERY, lq, q.device, workspace)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, lq), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_query(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), lq, _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_cache), _ptr(v_cache), k_cache.shape[1], _ptr(o), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream()), "star_attn_phase2_query")
    return o, lse


def phase2_decode(q, k, v, k_ctx, v_ctx, k_cache, v_cache, cache_len: int, block_size: int,
                  scale: Optional[float] = None, o=None, lse=None, workspace=None):
    """One decode step: q [b, 1, Hq, d], k/v [b, 1, Hkv, d]; the token's KV is appended at
    cache row cache_len and it attends to context + cache rows 0..cache_len."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx"),
                 (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n, 4)
    b, _, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    workspace = _ws(shape, STAR_PHASE2_DECODE, 1, q.device, workspace)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, 1), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_decode(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_cache),
        _ptr(v_cache), int(cache_len), k_cache.shape[1], _ptr(o), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream()), "star_attn_phase2_decode")
    return o, lse


def _page_pool(k_pages, v_pages, page_table):
    for t, n in ((k_pages, "k_pages"), (v_pages, "v_pages")):
        _bf16(t, n, 4)
    if k_pages.shape != v_pages.shape:
        raise ValueError("k_pages and v_pages must have the same shape")
    if (not isinstance(page_table, torch.Tensor) or page_table.dtype != torch.int32
            or page_table.dim() != 2 or not page_table.is_contiguous()
            or page_table.device != k_pages.device):
        raise TypeError("page_table must be a contiguous int32 [batch, max_pages] tensor "
                        "on the pool's device")
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    return page_size, num_pages, page_table.shape[1]


def phase2_query_paged(q, k, v, k_ctx, v_ctx, k_pages, v_pages, page_table, block_size: int,
                       scale: Optional[float] = None, o=None, lse=None, workspace=None):
    """phase2_query() with the query-local cache in a page pool: k_pages/v_pages
    [num_pages, page_size, Hkv, d] bf16, page_table [b, max_pages] int32; cache row r of
    sequence i lives in row r % page_size of page page_table[i, r // page_size]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx")):
        _bf16(t, n, 4)
    page_size, num_pages, max_pages = _page_pool(k_pages, v_pages, page_table)
    b, lq, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    workspace = _ws(shape, STAR_PHASE2_QUERY, lq, q.device, workspace)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, lq), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_query_paged(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), lq, _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_pages), _ptr(v_pages), page_size, num_pages, _ptr(page_table), max_pages,
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream()),
        "star_attn_phase2_query_paged")
    return o, lse


def phase2_decode_paged(q, k, v, k_ctx, v_ctx, k_pages, v_pages, page_table, cache_len: int,
                        block_size: int, scale: Optional[float] = None, o=None, lse=None,
                        workspace=None):
    """phase2_decode() with the query-local cache in a page pool (see phase2_query_paged)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx")):
        _bf16(t, n, 4)
    page_size, num_pages, max_pages = _page_pool(k_pages, v_pages, page_table)
    b, _, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    workspace = _ws(shape, STAR_PHASE2_DECODE, 1, q.device, workspace)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, 1), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_decode_paged(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_pages), _ptr(v_pages), page_size, num_pages, _ptr(page_table), max_pages,
        int(cache_len), _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream()),
        "star_attn_phase2_decode_paged")
    return o, lse


def fused_decode_workspace(batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
                           device, scale: Optional[float] = None) -> torch.Tensor:
    """A zeroed workspace for phase2_decode_fused() (reusable across its steps)."""
    shape = make_shape(batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size, scale)
    need = workspace_bytes(shape, STAR_PHASE2_DECODE_FUSED)
    if need == 0:
        raise ValueError("unsupported shape")
    return torch.zeros(need, dtype=torch.uint8, device=device)


def phase2_decode_fused(q, k, v, k_ctx, v_ctx, k_cache, v_cache, cache_len: int,
                        block_size: int, scale: Optional[float] = None, o=None, lse=None,
                        workspace=None):
    """phase2_decode() as one kernel (partials + last-CTA merge). `workspace` must come
    from fused_decode_workspace() (zeroed once, left zeroed by every call); one is made
    when it is None."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx"),
                 (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n, 4)
    b, _, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    if workspace is None:
        workspace = fused_decode_workspace(b, hq, k_ctx.shape[2], d, k_ctx.shape[1],
                                           block_size, q.device, scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, 1), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_decode_fused(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_cache),
        _ptr(v_cache), int(cache_len), k_cache.shape[1], _ptr(o), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream()), "star_attn_phase2_decode_fused")
    return o, lse


def phase2_query_varlen(q, k, v, k_ctx, v_ctx, cu_ctx, cu_q, k_cache, v_cache,
                        block_size: int, page_table=None, scale: Optional[float] = None,
                        o=None, lse=None, workspace=None):
    """Phase-2 query pass for sequences with their own context and query lengths:
    q [total_q, Hq, d], k/v [total_q, Hkv, d] packed with host offsets cu_q [b + 1];
    contexts k_ctx/v_ctx [total_ctx, Hkv, d] with cu_ctx [b + 1]; caches [b, cap, Hkv, d]
    (or page pools with page_table [b, max_pages]). Returns (o [total_q, Hq, d],
    lse [Hq, total_q])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_ctx, "k_ctx"), (v_ctx, "v_ctx")):
        _bf16(t, n, 3)
    cc, cvals = _cu_array(cu_ctx)
    cq, qvals = _cu_array(cu_q)
    b = len(cvals) - 1
    if len(qvals) != b + 1:
        raise ValueError("cu_ctx and cu_q need the same number of sequences")
    total_q, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[1], d, cvals[-1], block_size, scale)
    if workspace is None:
        need = int(lib().star_attn_query_varlen_workspace_bytes(ctypes.byref(shape), cc, cq))
        if need == 0:
            raise ValueError("unsupported shape or offsets")
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if page_table is not None:
        page_size, num_pages, max_pages = _page_pool(k_cache, v_cache, page_table)
        cap = 0
    else:
        _bf16(k_cache, "k_cache", 4)
        _bf16(v_cache, "v_cache", 4)
        page_size = num_pages = max_pages = 0
        cap = k_cache.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((hq, total_q), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_query_varlen(
        ctypes.byref(shape), cc, cq, _ptr(q), _ptr(k), _ptr(v), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_cache), _ptr(v_cache), cap, _ptr(page_table), page_size, num_pages, max_pages,
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream()),
        "star_attn_phase2_query_varlen")
    return o, lse


def phase2_partial(q, block_size: int, k_ctx=None, v_ctx=None, k=None, v=None, k_cache=None,
                   v_cache=None, cache_len: int = 0, scale: Optional[float] = None,
                   workspace=None):
    """One host's share of Phase 2 in the multi-host form: attention of the rows of
    q [b, rows, Hq, d] over this host's context (k_ctx/v_ctx [b, L, Hkv, d], all
    visible) and, on the query host, its query-local cache (k_cache/v_cache with the
    rows' own k/v: one row = a decode step appended at cache_len, several rows = the
    query tokens written to rows [0, rows)). Returns (o32 [b, rows, Hq, d] fp32,
    lse [b, Hq, rows]) for star_attn_lse_merge across hosts."""
    _bf16(q, "q", 4)
    b, rows, hq, d = q.shape
    if k_ctx is None and k_cache is None:
        raise ValueError("a host needs context keys, a cache, or both")
    if k_ctx is not None:
        _bf16(k_ctx, "k_ctx", 4)
        _bf16(v_ctx, "v_ctx", 4)
        hkv, L = k_ctx.shape[2], k_ctx.shape[1]
    else:
        hkv, L = k_cache.shape[2], 1
    if k_cache is not None:
        for t, n in ((k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
            _bf16(t, n, 4)
    shape = make_shape(b, hq, hkv, d, L, block_size, scale)
    if workspace is None:
        workspace = _ws(shape, STAR_PHASE2_DECODE if rows == 1 else STAR_PHASE2_QUERY, rows,
                        q.device, None)
    o32 = torch.empty((b, rows, hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((b, hq, rows), dtype=torch.float32, device=q.device)
    cap = 0 if k_cache is None else k_cache.shape[1]
    _check(lib().star_attn_phase2_partial(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), rows, _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_cache), _ptr(v_cache), int(cache_len), cap, _ptr(o32), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream()), "star_attn_phase2_partial")
    return o32, lse


def decode_varlen_workspace(batch, num_q_heads, num_kv_heads, head_dim, cu_ctx, block_size,
                            device, scale: Optional[float] = None) -> torch.Tensor:
    """A zeroed workspace for phase2_decode_varlen() with these context offsets."""
    cu, vals = _cu_array(cu_ctx)
    shape = make_shape(batch, num_q_heads, num_kv_heads, head_dim, vals[-1], block_size, scale)
    need = int(lib().star_attn_decode_varlen_workspace_bytes(ctypes.byref(shape), cu))
    if need == 0:
        raise ValueError("unsupported shape or offsets")
    return torch.zeros(need, dtype=torch.uint8, device=device)


def phase2_decode_varlen(q, k, v, k_ctx, v_ctx, cu_ctx, k_cache, v_cache, cache_lens,
                         block_size: int, page_table=None, scale: Optional[float] = None,
                         o=None, lse=None, workspace=None):
    """One decode step for a batch of sequences at different lengths: q [b, 1, Hq, d],
    k/v [b, 1, Hkv, d]; packed contexts k_ctx/v_ctx [total, Hkv, d] with host offsets
    cu_ctx [b + 1]; caches [b, cap, Hkv, d] (or page pools with page_table [b, max_pages])
    holding cache_lens[i] rows (host). Appends each new token's KV at row cache_lens[i]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n, 4)
    _bf16(k_ctx, "k_ctx", 3)
    _bf16(v_ctx, "v_ctx", 3)
    cu, vals = _cu_array(cu_ctx)
    lens, lvals = _cu_array(cache_lens)
    b, _, hq, d = q.shape
    if len(vals) != b + 1 or len(lvals) != b:
        raise ValueError("cu_ctx needs batch + 1 offsets and cache_lens batch entries")
    shape = make_shape(b, hq, k_ctx.shape[1], d, vals[-1], block_size, scale)
    if workspace is None:
        workspace = decode_varlen_workspace(b, hq, k_ctx.shape[1], d, vals, block_size, q.device,
                                            scale)
    if page_table is not None:
        page_size, num_pages, max_pages = _page_pool(k_cache, v_cache, page_table)
        cap = 0
    else:
        _bf16(k_cache, "k_cache", 4)
        _bf16(v_cache, "v_cache", 4)
        page_size = num_pages = max_pages = 0
        cap = k_cache.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, hq, 1), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_phase2_decode_varlen(
        ctypes.byref(shape), cu, lens, _ptr(q), _ptr(k), _ptr(v), _ptr(k_ctx), _ptr(v_ctx),
        _ptr(k_cache), _ptr(v_cache), cap, _ptr(page_table), page_size, num_pages, max_pages,
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _stream()),
        "star_attn_phase2_decode_varlen")
    return o, lse


def lse_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor):
    """o_parts [S, b, T, H, d] fp32, lse_parts [S, b, H, T] fp32 -> (o bf16 [b, T, H, d], lse)."""
    S, b, T, H, d = o_parts.shape
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise TypeError("partials must be float32")
    o_parts = o_parts.contiguous()
    lse_parts = lse_parts.contiguous()
    o = torch.empty((b, T, H, d), dtype=torch.bfloat16, device=o_parts.device)
    lse = torch.empty((b, H, T), dtype=torch.float32, device=o_parts.device)
    _check(lib().star_attn_lse_merge(_ptr(o_parts), _ptr(lse_parts), S, b, T, H, d, _ptr(o),
                                     _ptr(lse), _stream()), "star_attn_lse_merge")
    return o, lse


def simple_phase1(q, k, v, block_size: int, scale: Optional[float] = None):
    """Cross-check kernel (one warp per row) for Phase 1; same contract as phase1()."""
    shape = _ctx_shape(q, k, block_size, scale)
    b, L, hq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((b, hq, L), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_simple_phase1(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                         _ptr(lse), _stream()), "star_attn_simple_phase1")
    return o, lse


def simple_phase2(q, k_ctx, v_ctx, k_cache, v_cache, block_size: int, visible_base: int,
                  causal: bool, scale: Optional[float] = None):
    """Cross-check kernel for Phase 2: row r sees all context keys and cache rows
    0..visible_base + (r if causal else 0). The cache must already hold those rows."""
    b, rows, hq, d = q.shape
    shape = make_shape(b, hq, k_ctx.shape[2], d, k_ctx.shape[1], block_size, scale)
    o = torch.empty_like(q)
    lse = torch.empty((b, hq, rows), dtype=torch.float32, device=q.device)
    _check(lib().star_attn_simple_phase2(
        ctypes.byref(shape), _ptr(q), rows, _ptr(k_ctx), _ptr(v_ctx), _ptr(k_cache),
        _ptr(v_cache), k_cache.shape[1], visible_base, 1 if causal else 0, _ptr(o), _ptr(lse),
        _stream()), "star_attn_simple_phase2")
    return o, lse


def device_status() -> int:
    """Synchronise the current stream and return (and clear) the device status."""
    return int(lib().star_attn_get_device_status(_stream()))


def selftest_wait_timeout(wait_ns: int = 20_000_000) -> None:
    _check(lib().star_attn_selftest_wait_timeout(int(wait_ns), _stream()),
           "star_attn_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor) -> torch.Tensor:
    """The FMA-pipe 2^x of the softmax, applied to a float32 CUDA tensor."""
    if not x.is_cuda or x.dtype != torch.float32:
        raise TypeError("x must be a float32 CUDA tensor")
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(lib().star_attn_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream()),
           "star_attn_selftest_exp2")
    return y


def selftest_read(buf: torch.Tensor, sink: torch.Tensor, ctas: int) -> None:
    """Stream every byte of the CUDA tensor `buf` once (read-only bandwidth probe);
    `sink` is an int32 CUDA tensor of at least `ctas` elements."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise TypeError("buf must be a contiguous CUDA tensor")
    if sink.dtype != torch.int32 or sink.numel() < ctas or not sink.is_cuda:
        raise TypeError("sink must be an int32 CUDA tensor with ctas elements")
    _check(lib().star_attn_selftest_read(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink),
                                         int(ctas), _stream()), "star_attn_selftest_read")


def debug_build() -> bool:
    """Whether the loaded library was built with -DSTAR_DEBUG (index checks)."""
    return bool(lib().star_attn_debug_build())


def debug_record():
    """(refusals, source line, index, limit) of the first index a debug build's
    checks refused since the last call (zeros if none); synchronises the stream."""
    out = (ctypes.c_int64 * 4)()
    _check(lib().star_attn_debug_record(out, _stream()), "star_attn_debug_record")
    return tuple(int(v) for v in out)


def selftest_bounds(out: torch.Tensor, n: int) -> None:
    """Check index n against limit n with the kernels' store check (out: int32 CUDA
    tensor with at least n + 1 elements)."""
    if out.dtype != torch.int32 or not out.is_cuda or out.numel() < n + 1:
        raise TypeError("out must be an int32 CUDA tensor with n + 1 elements")
    _check(lib().star_attn_selftest_bounds(_ptr(out), int(n), _stream()), "star_attn_selftest_bounds")


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().star_attn_launch_count())


def version() -> str:
    return lib().star_attn_version().decode()


class StarAttentionLayer:
    """One attention layer's Star Attention state on one GPU: the context KV from
    Phase 1, the query-local cache, and the Phase-2 workspace (allocated once).

        layer = StarAttentionLayer(batch, Hq, Hkv, d, ctx_len, block_size, cache_capacity)
        o_ctx = layer.prefill(q, k, v)          # Phase 1; keeps k, v as the context KV
        o_q = layer.query(q_q, k_q, v_q)        # Phase 2, query tokens
        o_t = layer.decode(q_t, k_t, v_t)       # Phase 2, one decode step (repeat)
    """

    def __init__(self, batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
                 cache_capacity, device="cuda", scale: Optional[float] = None,
                 fused_decode: bool = True):
        self.shape = make_shape(batch, num_q_heads, num_kv_heads, head_dim, ctx_len, block_size,
                                scale)
        self.block_size = block_size
        self.scale = scale
        self.k_cache = torch.empty((batch, cache_capacity, num_kv_heads, head_dim),
                                   dtype=torch.bfloat16, device=device)
        self.v_cache = torch.empty_like(self.k_cache)
        self.cache_len = 0
        self.k_ctx = self.v_ctx = None
        # Decode steps run as one kernel each (partials + last-CTA merge) unless
        # fused_decode is False (partial kernel, then a merge kernel).
        self.fused_decode = fused_decode
        if fused_decode:
            self.ws_decode = fused_decode_workspace(batch, num_q_heads, num_kv_heads, head_dim,
                                                    ctx_len, block_size, device, scale)
        else:
            self.ws_decode = torch.empty(
                max(256, workspace_bytes(self.shape, STAR_PHASE2_DECODE)), dtype=torch.uint8,
                device=device)
        self.ws_query = None

    def prefill(self, q, k, v, o=None, lse=None):
        self.k_ctx, self.v_ctx = k, v
        self.cache_len = 0
        return phase1(q, k, v, self.block_size, self.scale, o=o, lse=lse)

    def query(self, q, k, v, o=None, lse=None):
        lq = q.shape[1]
        need = workspace_bytes(self.shape, STAR_PHASE2_QUERY, lq)
        if self.ws_query is None or self.ws_query.numel() < need:
            self.ws_query = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
        out = phase2_query(q, k, v, self.k_ctx, self.v_ctx, self.k_cache, self.v_cache,
                           self.block_size, self.scale, o=o, lse=lse, workspace=self.ws_query)
        self.cache_len = lq
        return out

    def decode(self, q, k, v, o=None, lse=None):
        fn = phase2_decode_fused if self.fused_decode else phase2_decode
        out = fn(q, k, v, self.k_ctx, self.v_ctx, self.k_cache, self.v_cache, self.cache_len,
                 self.block_size, self.scale, o=o, lse=lse, workspace=self.ws_decode)
        self.cache_len += 1
        return out
