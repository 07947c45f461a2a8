"""Paged query-local cache: the query pass and decode steps with the cache rows in a
page pool give the same bytes as with a contiguous cache (same kernels, same split
plan, same summation order), match the oracle, and land every appended row in the
page the table names. Pools start filled with NaN, so any read of a row that was
never written, or of another sequence's page, shows up in the outputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity_util import check_rows, to_np

pytestmark = pytest.mark.gpu


def sa():
    import block_sparse_attention_phase_b200 as m
    return m


def _pool(num_pages, page_size, hkv, d):
    k = torch.full((num_pages, page_size, hkv, d), float("nan"), dtype=torch.bfloat16,
                   device="cuda")
    return k, torch.full_like(k, float("nan"))


def _table(b, max_pages, num_pages, seed):
    """Distinct pages for every (sequence, slot), in a shuffled order."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.randperm(num_pages, generator=g)[: b * max_pages]
    return ids.view(b, max_pages).to(torch.int32).cuda()


def _gather(pool, table, rows):
    """Rows [0, rows) of every sequence, read back through the page table."""
    P = pool.shape[1]
    out = []
    for i in range(table.shape[0]):
        pages = [pool[int(table[i, j])] for j in range((rows + P - 1) // P)]
        out.append(torch.cat(pages, 0)[:rows])
    return torch.stack(out)


PAGED = [
    # b, Hq, Hkv, d, L, B, Lq, T, page_size
    (1, 4, 2, 128, 1000, 300, 126, 4, 128),   # decode fills page 0 and opens page 1
    (1, 4, 2, 128, 600, 256, 128, 2, 128),    # the first decode step opens a page
    (2, 8, 1, 64, 700, 256, 130, 3, 128),     # query rows span two pages; batch 2, G 8
    (1, 16, 4, 128, 384, 128, 300, 2, 256),   # three query tiles, 256-row pages
    (2, 4, 4, 64, 513, 512, 5, 3, 384),       # one page per sequence
]


@pytest.mark.parametrize("case", PAGED, ids=lambda c: "x".join(map(str, c)))
def test_paged_matches_contiguous_and_oracle(case):
    b, hq, hkv, d, L, B, lq, T, P = case
    m = sa()
    w = workloads.Workload("paged", b, hq, hkv, d, L, B, lq, T, 0, 11)
    x = workloads.make_inputs(w, device="cuda")
    cap = lq + T
    max_pages = (cap + P - 1) // P + 1
    num_pages = b * max_pages + 3
    kp, vp = _pool(num_pages, P, hkv, d)
    table = _table(b, max_pages, num_pages, seed=b * 1000 + lq)
    kc = torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))

    # ---- query pass
    o_c, l_c = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"],
                              kc, vc, B)
    o_p, l_p = m.phase2_query_paged(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"],
                                    x["v_ctx"], kp, vp, table, B)
    assert torch.equal(o_p, o_c) and torch.equal(l_p, l_c)
    rq, rql = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                  to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(o_p), rq, to_np(l_p), rql, f"paged query {case}")
    assert torch.equal(_gather(kp, table, lq), x["k_qry"])
    assert torch.equal(_gather(vp, table, lq), x["v_qry"])

    # ---- decode steps
    k_cache = np.zeros((b, cap, hkv, d))
    v_cache = np.zeros((b, cap, hkv, d))
    k_cache[:, :lq] = to_np(x["k_qry"])
    v_cache[:, :lq] = to_np(x["v_qry"])
    for t in range(T):
        args = (x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"], x["v_ctx"])
        od_c, ld_c = m.phase2_decode(*args, kc, vc, lq + t, B)
        od_p, ld_p = m.phase2_decode_paged(*args, kp, vp, table, lq + t, B)
        assert torch.equal(od_p, od_c) and torch.equal(ld_p, ld_c), f"decode t={t}"
        ro, rl, k_cache, v_cache = oracle.phase2_decode(
            to_np(x["q_dec"][t]), to_np(x["k_dec"][t]), to_np(x["v_dec"][t]),
            to_np(x["k_ctx"]), to_np(x["v_ctx"]), k_cache, v_cache, lq + t)
        check_rows(to_np(od_p), ro, to_np(ld_p), rl, f"paged decode {case} t={t}")
    rows = lq + T
    assert torch.equal(_gather(kp, table, rows), kc[:, :rows])
    assert torch.equal(_gather(vp, table, rows), vc[:, :rows])
    # pages no sequence owns were never touched
    owned = set(table.flatten().tolist())
    for pg in range(num_pages):
        if pg not in owned:
            assert torch.isnan(kp[pg].float()).all() and torch.isnan(vp[pg].float()).all()
    assert m.device_status() == 0


def test_paged_cache_full_and_bad_page_ids():
    m = sa()
    w = workloads.Workload("paged", 1, 4, 2, 64, 300, 128, 4, 1, 0, 5)
    x = workloads.make_inputs(w, device="cuda")
    kp, vp = _pool(4, 128, 2, 64)
    one = torch.tensor([[2]], dtype=torch.int32, device="cuda")
    m.phase2_query_paged(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kp, vp,
                         one, 128)
    args = (x["q_dec"][0], x["k_dec"][0], x["v_dec"][0], x["k_ctx"], x["v_ctx"])
    with pytest.raises(m.StarAttnError, match="CACHE_FULL"):
        m.phase2_decode_paged(*args, kp, vp, one, 128, 128)  # row 128 needs a second page
    # A page id outside the pool: the append is refused and flagged, nothing is written
    # outside the pool, and the step's reads of that page return zeros.
    for bad in (4, -1):
        before_k, before_v = kp.clone(), vp.clone()
        tbl = torch.tensor([[2, bad]], dtype=torch.int32, device="cuda")
        m.phase2_decode_paged(*args, kp, vp, tbl, 128, 128)
        assert m.device_status() == 5  # bounds flag -> STAR_ERR_CUDA, then cleared
        assert m.device_status() == 0
        assert torch.equal(kp.view(torch.int16), before_k.view(torch.int16))
        assert torch.equal(vp.view(torch.int16), before_v.view(torch.int16))
