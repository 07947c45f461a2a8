"""A seeded sweep of small random shapes through every call of the path (Phase 1,
the query pass, fused and two-kernel decode steps) against the
oracle: group sizes 1-8, head dims 64 and 128, ragged blocks and tiles, blocks
shorter and longer than a tile, contexts shorter than a block."""
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


def random_cases(n, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        hkv = int(rng.choice([1, 2]))
        G = int(rng.choice([1, 2, 4, 8]))
        d = int(rng.choice([64, 128]))
        L = int(rng.integers(1, 2500))
        B = int(rng.integers(1, L + 200))
        lq = int(rng.integers(1, 150))
        b = int(rng.choice([1, 2]))
        cases.append((b, hkv * G, hkv, d, L, B, lq, 2))
    return cases


CASES = random_cases(10)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_random_shape_through_every_call(case):
    b, hq, hkv, d, L, B, lq, T = case
    m = sa()
    w = workloads.Workload("sweep", b, hq, hkv, d, L, B, lq, T, 0, sum(case))
    x = workloads.make_inputs(w, device="cuda")
    o, lse = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], B)
    ro, rl = oracle.phase1(to_np(x["q_ctx"]), to_np(x["k_ctx"]), to_np(x["v_ctx"]), B)
    check_rows(to_np(o), ro, to_np(lse), rl, f"phase1 {case}")
    cap = lq + T
    caches = [torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
              for _ in range(4)]
    kc, vc, kc2, vc2 = caches
    oq, lql = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc, B)
    rq, rql = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                  to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(oq), rq, to_np(lql), rql, f"query {case}")
    kc2.copy_(kc)
    vc2.copy_(vc)
    k_ref = np.zeros((b, cap, hkv, d))
    v_ref = np.zeros((b, cap, hkv, d))
    k_ref[:, :lq], v_ref[:, :lq] = to_np(x["k_qry"]), to_np(x["v_qry"])
    ws = m.fused_decode_workspace(b, hq, hkv, d, L, B, "cuda")
    for t in range(T):
        args = (x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"], x["v_ctx"])
        of, lf = m.phase2_decode_fused(*args, kc, vc, lq + t, B, workspace=ws)
        os_, ls = m.phase2_decode(*args, kc2, vc2, lq + t, B)
        rod, rld, k_ref, v_ref = oracle.phase2_decode(
            to_np(x["q_dec"][t]), to_np(x["k_dec"][t]), to_np(x["v_dec"][t]), to_np(x["k_ctx"]),
            to_np(x["v_ctx"]), k_ref, v_ref, lq + t)
        check_rows(to_np(of), rod, to_np(lf), rld, f"fused decode {case} t={t}")
        check_rows(to_np(os_), rod, to_np(ls), rld, f"two-kernel decode {case} t={t}")
    assert torch.equal(kc[:, :lq + T], kc2[:, :lq + T])
    assert m.device_status() == 0
