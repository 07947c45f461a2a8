"""Varlen batches: sequences of different lengths packed along the token axis.
Every sequence must come out exactly as if it were run alone (bit-equal to a
batch-1 call of the uniform entry point) and match the oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import check_rows, to_np

pytestmark = pytest.mark.gpu


def sa():
    import block_sparse_attention_phase_b200 as m
    return m


def packed(lens, hq, hkv, d, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    total = sum(lens)
    mk = lambda h: (torch.randn(total, h, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    return mk(hq), mk(hkv), mk(hkv), cu


CASES = [
    # lens, Hq, Hkv, d, B
    ([700, 0, 300, 1300, 129, 1], 4, 2, 128, 512),   # ragged, empty, shorter than B
    ([513, 1024, 77], 8, 1, 64, 256),                # G = 8
    ([400, 900], 2, 2, 64, 128),                     # G = 1: two q-tiles per CTA
    ([5, 3, 1, 8], 4, 4, 128, 4),                    # blocks shorter than a tile
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[0])) + f"_g{c[1]//c[2]}_d{c[3]}")
def test_phase1_varlen_matches_oracle_and_alone(case):
    lens, hq, hkv, d, B = case
    m = sa()
    q, k, v, cu = packed(lens, hq, hkv, d, seed=sum(lens))
    o, lse = m.phase1_varlen(q, k, v, cu, B)
    ro, rl = oracle.phase1_varlen(to_np(q), to_np(k), to_np(v), cu, B)
    check_rows(to_np(o), ro, to_np(lse), rl, f"varlen {case}")
    for a, e in zip(cu[:-1], cu[1:]):
        if e == a:
            continue
        oa, la = m.phase1(q[None, a:e].contiguous(), k[None, a:e].contiguous(),
                          v[None, a:e].contiguous(), B)
        assert torch.equal(o[a:e], oa[0]) and torch.equal(lse[:, a:e], la[0])
    assert m.device_status() == 0


def test_phase1_varlen_long_sequences_equal_alone():
    """Llama-8B heads, three long documents of unequal length in one launch."""
    m = sa()
    lens = [9000, 3000, 20000]
    q, k, v, cu = packed(lens, 32, 8, 128, seed=5)
    o, lse = m.phase1_varlen(q, k, v, cu, 4096)
    for a, e in zip(cu[:-1], cu[1:]):
        oa, la = m.phase1(q[None, a:e].contiguous(), k[None, a:e].contiguous(),
                          v[None, a:e].contiguous(), 4096)
        assert torch.equal(o[a:e], oa[0]) and torch.equal(lse[:, a:e], la[0])
    # and a sampled oracle check on the last rows of the longest sequence, head 5
    a, e = cu[2], cu[3]
    rows = np.array([0, 1, 4095, 4096, 4097, 8191, 16383, 19999])
    ro, rl = oracle.phase1_head(to_np(q[a:e, 5]), to_np(k[a:e, 1]), to_np(v[a:e, 1]), 4096,
                                oracle.default_scale(128), rows)
    check_rows(to_np(o[a + rows, 5]), ro, to_np(lse[5, a + rows]), rl, "varlen long")
    assert m.device_status() == 0


DEC_CASES = [
    # ctx lens, cache lens, Hq, Hkv, d, B, paged page size (0: contiguous)
    ([3000, 0, 700, 9000], [5, 0, 17, 130], 8, 2, 128, 1024, 0),
    ([3000, 0, 700, 9000], [5, 0, 127, 130], 8, 2, 128, 1024, 128),
    ([513, 2048], [64, 3], 8, 1, 64, 512, 0),           # G = 8
    ([4096, 2048], [3, 5], 8, 1, 128, 512, 0),          # G = 8, d 128: 65 splits, merge in 4 passes
    ([40000, 100, 12000], [1, 2, 3], 32, 8, 128, 4096, 256),
]


@pytest.mark.parametrize("case", DEC_CASES, ids=lambda c: f"{len(c[0])}seq_g{c[2]//c[3]}_d{c[4]}_p{c[6]}")
def test_decode_varlen_matches_oracle(case):
    ctx_lens, lens0, hq, hkv, d, B, P = case
    m = sa()
    b = len(ctx_lens)
    T = 3
    g = torch.Generator(device="cpu").manual_seed(len(ctx_lens) * 7 + d)
    rnd = lambda *shape: (torch.randn(*shape, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    cu = [0]
    for n in ctx_lens:
        cu.append(cu[-1] + n)
    kc, vc = rnd(cu[-1], hkv, d), rnd(cu[-1], hkv, d)
    cap = max(lens0) + T
    k_rows, v_rows = rnd(b, cap, hkv, d), rnd(b, cap, hkv, d)  # rows [0, lens0[i]) are valid
    if P:
        max_pages = (cap + P - 1) // P
        num_pages = b * max_pages + 2
        gp = torch.Generator().manual_seed(3)
        table = torch.randperm(num_pages, generator=gp)[: b * max_pages].view(b, max_pages)
        table = table.to(torch.int32).cuda()
        kp = torch.zeros((num_pages, P, hkv, d), dtype=torch.bfloat16, device="cuda")
        vp = torch.zeros_like(kp)
        for i in range(b):
            for r in range(lens0[i]):
                kp[int(table[i, r // P]), r % P] = k_rows[i, r]
                vp[int(table[i, r // P]), r % P] = v_rows[i, r]
        kcache, vcache = kp, vp
    else:
        table = None
        kcache = torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        vcache = torch.full_like(kcache, float("nan"))
        for i in range(b):
            kcache[i, :lens0[i]] = k_rows[i, :lens0[i]]
            vcache[i, :lens0[i]] = v_rows[i, :lens0[i]]
    ws = m.decode_varlen_workspace(b, hq, hkv, d, cu, B, "cuda")
    k_ref = np.zeros((b, cap, hkv, d))
    v_ref = np.zeros((b, cap, hkv, d))
    for i in range(b):
        k_ref[i, :lens0[i]] = to_np(k_rows[i, :lens0[i]])
        v_ref[i, :lens0[i]] = to_np(v_rows[i, :lens0[i]])
    for t in range(T):
        lens = [n + t for n in lens0]
        q, k, v = rnd(b, 1, hq, d), rnd(b, 1, hkv, d), rnd(b, 1, hkv, d)
        o, lse = m.phase2_decode_varlen(q, k, v, kc, vc, cu, kcache, vcache, lens, B,
                                        page_table=table, workspace=ws)
        ro, rl, k_ref, v_ref = oracle.phase2_decode_varlen(
            to_np(q), to_np(k), to_np(v), to_np(kc), to_np(vc), cu, k_ref, v_ref, lens)
        check_rows(to_np(o), ro, to_np(lse), rl, f"decode varlen {case} t={t}")
        # the counters (the workspace's last 256-byte-aligned segment) are back at zero
        seg = (4 * b * hkv + 255) // 256 * 256
        ctr = ws[ws.numel() - seg: ws.numel() - seg + 4 * b * hkv].view(torch.int32)
        assert int(ctr.abs().sum()) == 0
        for i in range(b):  # the new row landed in sequence i's cache only
            if P:
                row = kcache[int(table[i, lens[i] // P]), lens[i] % P]
            else:
                row = kcache[i, lens[i]]
            assert torch.equal(row, k[i, 0])
    assert m.device_status() == 0


QRY_CASES = [
    # ctx lens, query lens, Hq, Hkv, d, B, page size (0: contiguous)
    ([3000, 0, 700, 9000], [5, 3, 0, 130], 8, 2, 128, 1024, 0),
    ([3000, 700, 9000], [200, 1, 64], 8, 2, 128, 1024, 256),
    ([513, 2048], [40, 17], 8, 1, 64, 512, 0),          # G = 8
]


@pytest.mark.parametrize("case", QRY_CASES, ids=lambda c: f"{len(c[0])}seq_g{c[2]//c[3]}_d{c[4]}_p{c[6]}")
def test_query_varlen_then_decode(case):
    """Varlen query pass against the oracle (NaN-filled caches), then a varlen decode
    step on the caches it wrote, against the oracle again."""
    ctx_lens, q_lens, hq, hkv, d, B, P = case
    m = sa()
    b = len(ctx_lens)
    g = torch.Generator(device="cpu").manual_seed(sum(ctx_lens) + d)
    rnd = lambda *shape: (torch.randn(*shape, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    cu_c, cu_q = [0], [0]
    for n in ctx_lens:
        cu_c.append(cu_c[-1] + n)
    for n in q_lens:
        cu_q.append(cu_q[-1] + n)
    kc, vc = rnd(cu_c[-1], hkv, d), rnd(cu_c[-1], hkv, d)
    q, k, v = rnd(cu_q[-1], hq, d), rnd(cu_q[-1], hkv, d), rnd(cu_q[-1], hkv, d)
    cap = max(q_lens) + 2
    if P:
        max_pages = (cap + P - 1) // P
        num_pages = b * max_pages + 1
        table = torch.randperm(num_pages, generator=torch.Generator().manual_seed(1))[: b * max_pages]
        table = table.view(b, max_pages).to(torch.int32).cuda()
        kcache = torch.full((num_pages, P, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    else:
        table = None
        kcache = torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vcache = torch.full_like(kcache, float("nan"))
    o, lse = m.phase2_query_varlen(q, k, v, kc, vc, cu_c, cu_q, kcache, vcache, B, page_table=table)
    ro, rl = oracle.phase2_query_varlen(to_np(q), to_np(k), to_np(v), to_np(kc), to_np(vc), cu_c, cu_q)
    check_rows(to_np(o), ro, to_np(lse), rl, f"query varlen {case}")
    # each sequence alone through the uniform entry point agrees
    for i in range(b):
        a, e = cu_q[i], cu_q[i + 1]
        if e == a or cu_c[i + 1] == cu_c[i]:
            continue
        kci = torch.zeros((1, cap, hkv, d), dtype=torch.bfloat16, device="cuda")
        vci = torch.zeros_like(kci)
        oi, li = m.phase2_query(q[None, a:e].contiguous(), k[None, a:e].contiguous(),
                                v[None, a:e].contiguous(), kc[None, cu_c[i]:cu_c[i + 1]].contiguous(),
                                vc[None, cu_c[i]:cu_c[i + 1]].contiguous(), kci, vci, B)
        check_rows(to_np(o[a:e]), to_np(oi[0]).astype(np.float64), to_np(lse[:, a:e]),
                   to_np(li[0]).astype(np.float64), f"query varlen vs alone {i}")
    # then one decode step per sequence on the caches the query pass wrote
    qd, kd, vd = rnd(b, 1, hq, d), rnd(b, 1, hkv, d), rnd(b, 1, hkv, d)
    od, ld = m.phase2_decode_varlen(qd, kd, vd, kc, vc, cu_c, kcache, vcache, q_lens, B,
                                    page_table=table)
    k_ref = np.zeros((b, cap, hkv, d))
    v_ref = np.zeros((b, cap, hkv, d))
    for i in range(b):
        k_ref[i, :q_lens[i]] = to_np(k[cu_q[i]:cu_q[i + 1]])
        v_ref[i, :q_lens[i]] = to_np(v[cu_q[i]:cu_q[i + 1]])
    rod, rld, _, _ = oracle.phase2_decode_varlen(to_np(qd), to_np(kd), to_np(vd), to_np(kc),
                                                 to_np(vc), cu_c, k_ref, v_ref, q_lens)
    check_rows(to_np(od), rod, to_np(ld), rld, f"decode after query varlen {case}")
    assert m.device_status() == 0
