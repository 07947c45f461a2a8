"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every
symbol include/star_attn.h declares, sizes workspaces, and rejects bad arguments
before launching anything."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_phase_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    text = open(os.path.join(ROOT, "include", "star_attn.h")).read()
    return sorted(set(re.findall(r"STAR_ATTN_API\s+[\w\s\*]+?\b(star_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = sa.lib()
    names = header_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(sa.EXPORTED) == names


def test_version_and_status_strings():
    assert "sm_100a" in sa.version()
    L = sa.lib()
    for code in range(7):
        assert L.star_attn_status_string(code)
    assert L.star_attn_status_string(6) == b"device-side wait timed out"


def test_workspace_bytes():
    s = sa.make_shape(1, 32, 8, 128, 32768, 4096)
    assert sa.workspace_bytes(s, sa.STAR_PHASE1) == 0
    dec = sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE)
    q = sa.workspace_bytes(s, sa.STAR_PHASE2_QUERY, 64)
    # fp32 partial outputs + LSEs: (d + 1) floats per split per (row, head)
    assert dec >= 32 * 129 * 4 * 9 and dec % 256 == 0
    assert q >= 64 * dec // 2
    assert sa.workspace_bytes(s, sa.STAR_PHASE2_QUERY, 0) == 0
    bad = sa.make_shape(1, 32, 6, 128, 1024, 128)  # Hq % Hkv != 0
    assert sa.workspace_bytes(bad, sa.STAR_PHASE2_DECODE) == 0


def _call_phase1(shape, ptrs):
    L = sa.lib()
    p = [ctypes.c_void_p(x) for x in ptrs]
    return L.star_attn_phase1(ctypes.byref(shape) if shape is not None else None, *p, None)


FAKE = 1 << 20  # aligned, never dereferenced: every call below is rejected on the host


@pytest.mark.parametrize("shape_args,code", [
    ((1, 4, 3, 128, 100, 10), 1),    # Hq % Hkv != 0
    ((1, 4, 2, 96, 100, 10), 2),     # head_dim 96 unsupported
    ((1, 12, 4, 128, 100, 10), 2),   # GQA group 3 unsupported
    ((0, 4, 2, 128, 100, 10), 1),    # batch 0
    ((1, 4, 2, 128, 0, 10), 1),      # empty context
    ((1, 4, 2, 128, 100, 0), 1),     # block size 0
])
def test_phase1_rejects_bad_shapes(shape_args, code):
    assert _call_phase1(sa.make_shape(*shape_args), [FAKE, FAKE, FAKE, FAKE, FAKE]) == code


def test_phase1_rejects_null_and_misaligned():
    s = sa.make_shape(1, 4, 2, 128, 100, 10)
    assert _call_phase1(None, [FAKE] * 5) == 1
    assert _call_phase1(s, [0, FAKE, FAKE, FAKE, FAKE]) == 1
    assert _call_phase1(s, [FAKE + 2, FAKE, FAKE, FAKE, FAKE]) == 1
    assert _call_phase1(s, [FAKE, FAKE, FAKE, FAKE + 8, FAKE]) == 1  # misaligned o
    assert _call_phase1(s, [FAKE, FAKE, FAKE, FAKE, FAKE + 2]) == 1  # lse not 4-byte aligned


def test_phase2_rejects_cache_and_workspace_errors():
    L = sa.lib()
    s = sa.make_shape(1, 4, 2, 128, 100, 10)
    F = ctypes.c_void_p(FAKE)
    need = sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE)
    # decode: cache_len + 1 > capacity
    assert L.star_attn_phase2_decode(ctypes.byref(s), F, F, F, F, F, F, F, 8, 8, F, None, F,
                                     need, None) == 4
    # decode: workspace too small
    assert L.star_attn_phase2_decode(ctypes.byref(s), F, F, F, F, F, F, F, 3, 8, F, None, F,
                                     need - 1, None) == 3
    assert L.star_attn_phase2_decode(ctypes.byref(s), F, F, F, F, F, F, F, 3, 8, F, None, None,
                                     need, None) == 3
    # query: more query tokens than cache rows
    needq = sa.workspace_bytes(s, sa.STAR_PHASE2_QUERY, 16)
    assert L.star_attn_phase2_query(ctypes.byref(s), F, F, F, 16, F, F, F, F, 8, F, None, F,
                                    needq, None) == 4
    assert L.star_attn_phase2_query(ctypes.byref(s), F, F, F, 4, F, F, F, F, 8, F, None, F,
                                    0, None) == 3
    # merge: bad sizes
    assert L.star_attn_lse_merge(F, F, 0, 1, 1, 1, 128, F, None, None) == 1
    assert L.star_attn_lse_merge(F, F, 2, 1, 1, 1, 80, F, None, None) == 2


def test_binding_checks_tensors_before_calling():
    import torch
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sa.phase1(q, q, q, 4)  # CPU tensors are refused: there is no CPU path


def test_paged_entry_points_reject_bad_pools():
    L = sa.lib()
    s = sa.make_shape(1, 4, 2, 128, 100, 10)
    F = ctypes.c_void_p(FAKE)
    needd = sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE)
    needq = sa.workspace_bytes(s, sa.STAR_PHASE2_QUERY, 200)

    def dec(page_size, num_pages, table, max_pages, cache_len, ws=needd):
        return L.star_attn_phase2_decode_paged(ctypes.byref(s), F, F, F, F, F, F, F, page_size,
                                               num_pages, table, max_pages, cache_len, F, None,
                                               F, ws, None)

    def qry(lq, page_size, num_pages, table, max_pages, ws=needq):
        return L.star_attn_phase2_query_paged(ctypes.byref(s), F, F, F, lq, F, F, F, F,
                                              page_size, num_pages, table, max_pages, F, None,
                                              F, ws, None)

    T = ctypes.c_void_p(FAKE)
    assert dec(100, 4, T, 2, 0) == 1          # page size not a multiple of 128
    assert dec(64, 4, T, 2, 0) == 1
    assert dec(128, 0, T, 2, 0) == 1          # empty pool
    assert dec(128, 4, None, 2, 0) == 1       # no page table
    assert dec(128, 4, ctypes.c_void_p(FAKE + 2), 2, 0) == 1  # misaligned table
    assert dec(128, 4, T, 0, 0) == 1          # no page slots
    assert dec(128, 4, T, 2, 256) == 4        # row 256 needs a third page
    assert dec(128, 4, T, 2, 255, needd - 1) == 3
    assert qry(200, 128, 4, T, 1) == 4        # 200 rows need two pages
    assert qry(200, 256, 4, T, 1, 0) == 3     # fits one page, but no workspace
    assert qry(0, 128, 4, T, 2) == 1


def test_fused_decode_workspace_and_validation():
    L = sa.lib()
    s = sa.make_shape(2, 32, 8, 128, 32768, 4096)
    split = sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE)
    fused = sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE_FUSED)
    assert fused == split + 256  # one uint32 counter per (sequence, kv-head), 256-B aligned
    F = ctypes.c_void_p(FAKE)
    args = [F, F, F, F, F, F, F]
    assert L.star_attn_phase2_decode_fused(ctypes.byref(s), *args, 3, 8, F, None, F, split,
                                           None) == 3  # room for partials but not counters
    assert L.star_attn_phase2_decode_fused(ctypes.byref(s), *args, 8, 8, F, None, F, fused,
                                           None) == 4  # cache full
    assert L.star_attn_phase2_decode_fused(ctypes.byref(s), *args, -1, 8, F, None, F, fused,
                                           None) == 1


def test_phase1_varlen_rejects_bad_offsets():
    L = sa.lib()
    F = ctypes.c_void_p(FAKE)

    def call(cu, total, batch=None):
        n = len(cu) - 1 if batch is None else batch
        s = sa.make_shape(n, 4, 2, 128, total, 64)
        arr = (ctypes.c_int64 * len(cu))(*cu)
        return L.star_attn_phase1_varlen(ctypes.byref(s), arr, F, F, F, F, None, None)

    assert call([1, 5, 9], 9) == 1        # does not start at 0
    assert call([0, 5, 4], 4) == 1        # decreasing
    assert call([0, 5, 9], 10) == 1       # last offset != ctx_len
    assert call([0] + list(range(1, 130)), 129) == 2  # 129 sequences: more than 128
    s = sa.make_shape(2, 4, 2, 128, 9, 64)
    assert L.star_attn_phase1_varlen(ctypes.byref(s), None, F, F, F, F, None, None) == 1


def _plan(b, hkv, L, B, target):
    """The split plan the library documents: per (batch, kv-head), the query-local
    cache split plus context splits that are chunks of one block (at least one per
    block, at least 64 keys each), as many as bring the CTAs to about `target`."""
    B = min(B, L)
    n = -(-L // B)
    spb = max(1, (target // (b * hkv) - 1) // n)
    chunk = -(-B // spb)
    if chunk < 64:
        chunk = 64
        spb = -(-B // chunk)
    return n * spb + 1  # splits: context chunks + the cache


def _partial_bytes(splits, b, rows, hq, d):
    per = splits * b * rows * hq
    align = lambda x: (x + 255) // 256 * 256  # noqa: E731
    return align(per * d * 4) + align(per * 4)


@pytest.mark.parametrize("b,hq,hkv,d,L,B,lq", [
    (1, 32, 8, 128, 32768, 4096, 64),        # llama8b-32k: 16 context splits of 2048 + cache
    (1, 32, 8, 128, 1048576, 32768, 32),     # 1m: 4 x 32 q-rows in one tile pair
    (2, 64, 8, 128, 131072, 16384, 64),      # 70b-128k shape: G = 8
    (1, 4, 2, 64, 640, 256, 8),              # small: the 64-key minimum chunk binds
    (3, 8, 8, 128, 1000, 100000, 300),       # B clamped to L, G = 1, several q-tile pairs
])
def test_split_plans_match_their_rule(b, hq, hkv, d, L, B, lq):
    """Workspace sizes are the fp32 partials of exactly the planned splits: decode
    aims at 2 CTAs per SM, the query pass at one wave of (splits x q-tile pairs).
    Without a GPU the library plans for 148 SMs."""
    sms = 148
    s = sa.make_shape(b, hq, hkv, d, L, B)
    dec = _plan(b, hkv, L, B, 2 * sms)
    assert sa.workspace_bytes(s, sa.STAR_PHASE2_DECODE) == _partial_bytes(dec, b, 1, hq, d)
    pairs = (-(-(lq * (hq // hkv)) // 128) + 1) // 2
    qry = _plan(b, hkv, L, B, sms // pairs)
    assert sa.workspace_bytes(s, sa.STAR_PHASE2_QUERY, lq) == _partial_bytes(qry, b, lq, hq, d)
