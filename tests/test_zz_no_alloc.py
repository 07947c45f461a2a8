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
