"""The one-kernel decode step (split-KV partials whose last CTA per (sequence,
kv-head) merges the splits) against the oracle and against the two-kernel step:
every row, several shapes and steps in a row, the counter words back at zero
after every call, deterministic results, and CUDA-graph replays of the same
captured steps."""
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


def _counters(m, ws, w):
    """The counter words: the last b * Hkv uint32 of the partials region's end."""
    shape = m.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.ctx_len,
                         w.block_size)
    start = m.workspace_bytes(shape, m.STAR_PHASE2_DECODE)
    n = w.batch * w.num_kv_heads
    return ws[start:start + 4 * n].view(torch.int32)


CASES = [
    # b, Hq, Hkv, d, L, B, Lq, T
    (1, 2, 2, 64, 2048, 512, 16, 6),
    (1, 4, 2, 128, 1000, 300, 5, 3),
    (2, 8, 1, 64, 700, 256, 3, 3),
    (1, 2, 1, 64, 40, 1, 2, 2),          # 40 one-token blocks: 41 splits of one key
    (1, 8, 8, 128, 20000, 2500, 9, 3),   # G = 1, many splits per block
    (2, 64, 8, 128, 9000, 4096, 4, 2),   # G = 8, ragged last block
    (1, 64, 8, 128, 8192, 1024, 4, 2),   # G = 8, 33 splits: the merge stages them in 2 passes
    (1, 8, 1, 64, 2000, 1, 2, 2),        # 2001 splits: too many to fuse, runs unfused
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_fused_decode_matches_oracle_and_split_path(case):
    b, hq, hkv, d, L, B, lq, T = case
    m = sa()
    w = workloads.Workload("fused", b, hq, hkv, d, L, B, lq, T, 0, 21)
    x = workloads.make_inputs(w, device="cuda")
    cap = lq + T
    kc = torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc, B)
    kc2, vc2 = kc.clone(), vc.clone()
    ws = m.fused_decode_workspace(b, hq, hkv, d, L, B, "cuda")
    k_cache = np.zeros((b, cap, hkv, d))
    v_cache = np.zeros((b, cap, hkv, d))
    k_cache[:, :lq] = to_np(x["k_qry"])
    v_cache[:, :lq] = to_np(x["v_qry"])
    for t in range(T):
        args = (x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"], x["v_ctx"])
        of, lf = m.phase2_decode_fused(*args, kc2, vc2, lq + t, B, workspace=ws)
        assert int(_counters(m, ws, w).abs().sum()) == 0, "counters not reset"
        os_, ls = m.phase2_decode(*args, kc, vc, lq + t, B)
        ro, rl, k_cache, v_cache = oracle.phase2_decode(
            to_np(x["q_dec"][t]), to_np(x["k_dec"][t]), to_np(x["v_dec"][t]),
            to_np(x["k_ctx"]), to_np(x["v_ctx"]), k_cache, v_cache, lq + t)
        check_rows(to_np(of), ro, to_np(lf), rl, f"fused {case} t={t}")
        # same partials, merged in another order: within a bf16 rounding step
        diff = (of.float() - os_.float()).abs()
        assert float(diff.max()) <= 2.0 ** -7 * float(os_.float().abs().max()) + 1e-6
        assert float((lf - ls).abs().max()) <= 1e-5
        # deterministic: the same step again (its append rewrites the same row)
        of2, lf2 = m.phase2_decode_fused(*args, kc2, vc2, lq + t, B, workspace=ws)
        assert torch.equal(of, of2) and torch.equal(lf, lf2)
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    assert m.device_status() == 0


def test_fused_decode_graph_replays():
    """Captured steps replayed twice reuse the counters; results equal eager calls."""
    m = sa()
    b, hq, hkv, d, L, B, lq, T = 1, 32, 8, 128, 8192, 2048, 8, 4
    w = workloads.Workload("graph", b, hq, hkv, d, L, B, lq, T, 0, 3)
    x = workloads.make_inputs(w, device="cuda")
    cap = lq + T
    kc = torch.zeros((b, cap, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc, B)
    ws = m.fused_decode_workspace(b, hq, hkv, d, L, B, "cuda")
    o = torch.empty((T, b, 1, hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, b, hq, 1), dtype=torch.float32, device="cuda")

    def steps():
        for t in range(T):
            m.phase2_decode_fused(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"],
                                  x["v_ctx"], kc, vc, lq + t, B, o=o[t], lse=lse[t],
                                  workspace=ws)

    steps()
    torch.cuda.synchronize()
    o_eager, l_eager = o.clone(), lse.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            steps()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        o.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_eager) and torch.equal(lse, l_eager)
        assert int(_counters(m, ws, w).abs().sum()) == 0
    del g
    assert m.device_status() == 0
