"""The multi-host form's GPU pieces on one GPU: per-rank Phase 1 on [anchor ; own
blocks] is bit-identical to the rows of the single-GPU launch; per-rank Phase-2
partials (star_attn_phase2_partial) merged with star_attn_lse_merge match the
single-host query pass and decode steps and the oracle. The ranks are emulated
one after another (no rank waits on another); the collectives are covered by the
gloo tests."""
import math

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


@pytest.mark.parametrize("P", [1, 3])
def test_emulated_ranks_match_single_gpu(P):
    m = sa()
    b, hq, hkv, d, L, B, lq, T = 1, 8, 2, 128, 8192, 1024, 40, 2
    w = workloads.Workload("sharded", b, hq, hkv, d, L, B, lq, T, 0, 9)
    x = workloads.make_inputs(w, device="cuda")
    q, k, v = x["q_ctx"], x["k_ctx"], x["v_ctx"]
    o_full, l_full = m.phase1(q, k, v, B)
    n = math.ceil(L / B)
    ranges = [(min(r * n // P * B, L), min((r + 1) * n // P * B, L)) for r in range(P)]
    # ---- Phase 1 per rank
    ka, va = k[:, :B].contiguous(), v[:, :B].contiguous()  # what the anchor broadcast delivers
    for t0, t1 in ranges:
        sl = lambda t: t[:, t0:t1].contiguous()  # noqa: E731
        if t0 == 0:
            o, l = m.phase1(sl(q), sl(k), sl(v), B)
        else:
            o, l = m.phase1_anchored(sl(q), sl(k), sl(v), ka, va, B)
        assert torch.equal(o, o_full[:, t0:t1]) and torch.equal(l, l_full[..., t0:t1])
    # ---- Phase 2: the last rank is the query host
    cap = lq + T
    kc = torch.zeros((b, cap, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kref, vref = kc.clone(), vc.clone()

    def merged(qx, kx, vx, cache_len):
        parts = []
        for r, (t0, t1) in enumerate(ranges):
            host = r == P - 1
            parts.append(m.phase2_partial(
                qx, B, k_ctx=k[:, t0:t1].contiguous(), v_ctx=v[:, t0:t1].contiguous(),
                k=kx if host else None, v=vx if host else None, k_cache=kc if host else None,
                v_cache=vc if host else None, cache_len=cache_len))
        return m.lse_merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))

    oq, lqq = merged(x["q_qry"], x["k_qry"], x["v_qry"], 0)
    rq, rql = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], k, v, kref, vref, B)
    check_rows(to_np(oq), to_np(rq).astype(np.float64), to_np(lqq), to_np(rql).astype(np.float64),
               f"query P={P}")
    oo, ol = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]), to_np(k), to_np(v))
    check_rows(to_np(oq), oo, to_np(lqq), ol, f"query P={P} vs oracle")
    for t in range(T):
        od, ld = merged(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], lq + t)
        rd, rdl = m.phase2_decode(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], k, v, kref, vref,
                                  lq + t, B)
        check_rows(to_np(od), to_np(rd).astype(np.float64), to_np(ld), to_np(rdl).astype(np.float64),
                   f"decode P={P} t={t}")
    assert torch.equal(kc, kref) and torch.equal(vc, vref)
    assert m.device_status() == 0


@pytest.mark.parametrize("b,hq,hkv,d,L,B,t0", [
    (1, 8, 2, 128, 9000, 1024, 3072),   # G = 4; the last local block is ragged
    (2, 4, 4, 64, 2600, 640, 640),      # G = 1 (pairs of q-tiles of one head), batch 2
    (1, 4, 2, 128, 2100, 1024, 2048),   # a host holding only a short last block (52 < B rows)
    (1, 16, 2, 128, 1500, 300, 900),    # G = 8, B not a multiple of 128
])
def test_phase1_anchored_rows_equal_the_single_launch(b, hq, hkv, d, L, B, t0):
    """A host's blocks b_i.. (i > 0) with the anchor passed as its own buffer give
    exactly the rows the whole-context launch gives for them (same tiles, same
    order), and they match the oracle."""
    m = sa()
    w = workloads.Workload("anch", b, hq, hkv, d, L, B, 1, 1, 0, 11)
    x = workloads.make_inputs(w, device="cuda", parts=("ctx",))
    q, k, v = x["q_ctx"], x["k_ctx"], x["v_ctx"]
    o_full, l_full = m.phase1(q, k, v, B)
    ka, va = k[:, :B].contiguous(), v[:, :B].contiguous()
    o, l = m.phase1_anchored(q[:, t0:].contiguous(), k[:, t0:].contiguous(), v[:, t0:].contiguous(),
                             ka, va, B)
    assert torch.equal(o, o_full[:, t0:]) and torch.equal(l, l_full[..., t0:])
    rows = np.arange(t0, L)
    for bi in range(b):
        for h in (0, hq - 1):
            g = h // (hq // hkv)
            ro, rl = oracle.phase1_head(to_np(q[bi, :, h]), to_np(k[bi, :, g]), to_np(v[bi, :, g]), B,
                                        1.0 / math.sqrt(d), rows)
            check_rows(to_np(o[bi, :, h]), ro, to_np(l[bi, h]), rl, f"anchored b={bi} h={h}")
    assert m.device_status() == 0


def test_partial_without_context_or_cache_parts():
    """A host with no context (cache only) and a host with no cache (context only):
    their merge equals the query pass over both."""
    m = sa()
    b, hq, hkv, d, L, B, lq = 2, 4, 4, 64, 700, 256, 9
    w = workloads.Workload("parts", b, hq, hkv, d, L, B, lq, 1, 0, 4)
    x = workloads.make_inputs(w, device="cuda")
    cap = lq + 1
    kc = torch.zeros((b, cap, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    a = m.phase2_partial(x["q_qry"], B, k_ctx=x["k_ctx"], v_ctx=x["v_ctx"])
    c = m.phase2_partial(x["q_qry"], B, k=x["k_qry"], v=x["v_qry"], k_cache=kc, v_cache=vc)
    o, l = m.lse_merge(torch.stack([a[0], c[0]]), torch.stack([a[1], c[1]]))
    ro, rl = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                 to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(o), ro, to_np(l), rl, "context-only + cache-only")
    # the same for a decode step (one row)
    a = m.phase2_partial(x["q_dec"][0], B, k_ctx=x["k_ctx"], v_ctx=x["v_ctx"])
    c = m.phase2_partial(x["q_dec"][0], B, k=x["k_dec"][0], v=x["v_dec"][0], k_cache=kc,
                         v_cache=vc, cache_len=lq)
    o, l = m.lse_merge(torch.stack([a[0], c[0]]), torch.stack([a[1], c[1]]))
    kr = np.zeros((b, cap, hkv, d))
    vr = np.zeros_like(kr)
    kr[:, :lq], vr[:, :lq] = to_np(x["k_qry"]), to_np(x["v_qry"])
    rd, rdl, _, _ = oracle.phase2_decode(to_np(x["q_dec"][0]), to_np(x["k_dec"][0]),
                                         to_np(x["v_dec"][0]), to_np(x["k_ctx"]), to_np(x["v_ctx"]),
                                         kr, vr, lq)
    check_rows(to_np(o), rd, to_np(l), rdl, "decode: context-only + cache-only")
    assert m.device_status() == 0


def test_sharded_layer_single_rank():
    """The sharded layer with one rank (no process group) equals the plain layer."""
    from block_sparse_attention_phase_b200.sharded import ShardedStarAttention
    m = sa()
    b, hq, hkv, d, L, B, lq, T = 1, 8, 2, 128, 3000, 1024, 7, 2
    w = workloads.Workload("one", b, hq, hkv, d, L, B, lq, T, 0, 6)
    x = workloads.make_inputs(w, device="cuda")
    att = ShardedStarAttention(b, hq, hkv, d, L, B, lq + T)
    assert att.token_range() == (0, L)
    o, l = att.prefill(x["q_ctx"], x["k_ctx"], x["v_ctx"])
    ro, rl = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], B)
    assert torch.equal(o, ro) and torch.equal(l, rl)
    oq, _ = att.query(x["q_qry"], x["k_qry"], x["v_qry"])
    rq, _ = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(oq), rq, None, None, "sharded single-rank query")
    od, _ = att.decode(x["q_dec"][0], x["k_dec"][0], x["v_dec"][0])
    assert od.shape == (b, 1, hq, d)
    assert m.device_status() == 0
