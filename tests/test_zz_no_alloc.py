"""The allocation-free decode entry point against the workspace one.

star_attn_phase2_decode_noalloc serves callers that cannot allocate device
memory where they decode (a pooled allocator owns the GPU, cudaMalloc's implicit
synchronisation is not allowed, or a C caller has no allocator at hand). It keeps
its partials in a fixed array inside the library, so it must give the same
results as star_attn_phase2_decode with a caller workspace, call after call.
"""
import ctypes

import pytest
import torch

import workloads
from tests.parity_util import check_rows, to_np

pytestmark = pytest.mark.gpu


def _call_noalloc(sa, shape, q, k, v, kc, vc, k_cache, v_cache, cache_len, o, lse):
    return sa.lib().star_attn_phase2_decode_noalloc(
        ctypes.byref(shape), sa._ptr(q), sa._ptr(k), sa._ptr(v), sa._ptr(kc), sa._ptr(vc),
        sa._ptr(k_cache), sa._ptr(v_cache), cache_len, k_cache.shape[1], sa._ptr(o), sa._ptr(lse),
        sa._stream())


def test_noalloc_decode_matches_workspace_decode_twice():
    import block_sparse_attention_phase_b200 as sa
    w = workloads.Workload("noalloc", 2, 8, 2, 128, 3000, 1024, 5, 2, 0, 4)
    x = workloads.make_inputs(w, device="cuda")
    cap = 16
    kc_a = torch.zeros((2, cap, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc_a = torch.zeros_like(kc_a)
    sa.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc_a, vc_a, 1024)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    shape = sa.make_shape(2, 8, 2, 128, 3000, 1024)
    for t in range(2):  # two calls in a row: the shared array is reused
        o_ref, l_ref = sa.phase2_decode(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"],
                                        x["v_ctx"], kc_a, vc_a, 5 + t, 1024)
        o = torch.empty_like(o_ref)
        lse = torch.empty_like(l_ref)
        st = _call_noalloc(sa, shape, x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"],
                           x["v_ctx"], kc_b, vc_b, 5 + t, o, lse)
        assert st == 0, sa.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        check_rows(to_np(o), to_np(o_ref), to_np(lse), to_np(l_ref), f"noalloc t={t}")
        assert torch.equal(kc_b[:, 5 + t], x["k_dec"][t][:, 0])
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)
    assert sa.device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_array():
    import block_sparse_attention_phase_b200 as sa
    # 64 sequences x 64 q-heads x 129 floats for each split is far beyond 4 MiB
    shape = sa.make_shape(64, 64, 8, 128, 1 << 20, 1024)
    assert sa.workspace_bytes(shape, sa.STAR_PHASE2_DECODE) > (4 << 20)
    F = ctypes.c_void_p(1 << 20)
    st = sa.lib().star_attn_phase2_decode_noalloc(ctypes.byref(shape), F, F, F, F, F, F, F, 0, 8,
                                                  F, None, None)
    assert st == 3  # STAR_ERR_WORKSPACE, nothing launched


def test_noalloc_reports_unsupported_shapes_like_the_workspace_call():
    import block_sparse_attention_phase_b200 as sa
    # Shapes the library does not implement get STAR_ERR_UNSUPPORTED from both entry
    # points (checked before any pointer is looked at, so nothing is launched).
    F = ctypes.c_void_p(1 << 20)
    for shape in (sa.make_shape(1, 4, 2, 96, 4096, 1024),    # head_dim 96
                  sa.make_shape(1, 6, 2, 128, 4096, 1024)):  # GQA group of 3
        st_ws = sa.lib().star_attn_phase2_decode(ctypes.byref(shape), F, F, F, F, F, F, F, 0, 8,
                                                 F, None, F, 1 << 20, None)
        st = sa.lib().star_attn_phase2_decode_noalloc(ctypes.byref(shape), F, F, F, F, F, F, F,
                                                      0, 8, F, None, None)
        assert st_ws == 2 and st == 2, (st_ws, st)  # STAR_ERR_UNSUPPORTED
    bad = sa.make_shape(1, 4, 3, 128, 4096, 1024)  # Hq not a multiple of Hkv
    st = sa.lib().star_attn_phase2_decode_noalloc(ctypes.byref(bad), F, F, F, F, F, F, F, 0, 8,
                                                  F, None, None)
    assert st == 1  # STAR_ERR_INVALID_ARG


def test_noalloc_shape_that_just_fits_its_array():
    """The largest block count whose partials still fit the 4 MiB array runs and
    matches the workspace call (so the array's tail is in use); one block more is
    refused with STAR_ERR_WORKSPACE."""
    import block_sparse_attention_phase_b200 as sa
    b, hq, hkv, d, B = 2, 32, 8, 128, 256
    limit = 4 << 20
    n = 1
    while sa.workspace_bytes(sa.make_shape(b, hq, hkv, d, (n + 1) * B, B),
                             sa.STAR_PHASE2_DECODE) <= limit:
        n += 1
    L = n * B
    shape = sa.make_shape(b, hq, hkv, d, L, B)
    need = sa.workspace_bytes(shape, sa.STAR_PHASE2_DECODE)
    assert limit - 64 * 1024 < need <= limit, need
    w = workloads.Workload("noalloc-edge", b, hq, hkv, d, L, B, 3, 1, 0, 5)
    x = workloads.make_inputs(w, device="cuda")
    cap = 8
    kc_a = torch.zeros((b, cap, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc_a = torch.zeros_like(kc_a)
    sa.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc_a, vc_a, B)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    o_ref, l_ref = sa.phase2_decode(x["q_dec"][0], x["k_dec"][0], x["v_dec"][0], x["k_ctx"],
                                    x["v_ctx"], kc_a, vc_a, 3, B)
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    st = _call_noalloc(sa, shape, x["q_dec"][0], x["k_dec"][0], x["v_dec"][0], x["k_ctx"],
                       x["v_ctx"], kc_b, vc_b, 3, o, lse)
    assert st == 0, sa.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    check_rows(to_np(o), to_np(o_ref), to_np(lse), to_np(l_ref), "noalloc at the array's limit")
    # same kernels, same split plan: the two calls agree exactly
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)
    over = sa.make_shape(b, hq, hkv, d, L + B, B)
    assert sa.workspace_bytes(over, sa.STAR_PHASE2_DECODE) > limit
    st = _call_noalloc(sa, over, x["q_dec"][0], x["k_dec"][0], x["v_dec"][0], x["k_ctx"],
                       x["v_ctx"], kc_b, vc_b, 3, o, lse)
    assert st == 3  # STAR_ERR_WORKSPACE, nothing launched
    assert sa.device_status() == 0
