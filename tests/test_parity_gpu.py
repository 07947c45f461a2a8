"""GPU parity: the CUDA path (through the C-ABI) against the float64 CPU oracle.

Small shapes are compared row for row; they span several tiles, ragged last
blocks, one-block and one-token-block contexts, GQA groups 1/2/4/8, head_dim
64/128 and batch 2. The five named workloads run at full size in the launch
configuration the benchmark times; there the oracle checks sampled rows (block
edges, tile edges, planted rows, random rows) for Phase 1 and every row of
sampled heads for Phase 2.
"""
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


def make(b, hq, hkv, d, L, B, lq, T, seed=0, plants=0):
    w = workloads.Workload("case", b, hq, hkv, d, L, B, lq, T, plants, seed)
    return w, workloads.make_inputs(w, device="cuda")


SMALL = [
    # b, Hq, Hkv, d, L, B, Lq, T
    (1, 2, 2, 64, 2048, 512, 16, 8),     # the tiny workload
    (1, 4, 2, 128, 1000, 300, 5, 3),     # ragged last block, B not a tile multiple
    (2, 8, 1, 64, 700, 256, 3, 2),       # GQA group 8, batch 2
    (1, 4, 1, 128, 200, 512, 4, 2),      # L < B: one block, plain causal attention
    (1, 2, 2, 128, 512, 256, 1, 2),      # two blocks, Lq = 1
    (1, 2, 1, 64, 40, 1, 2, 2),          # B = 1: every block is one token
    (1, 4, 4, 128, 450, 100, 7, 2),      # B < tile
    (1, 2, 2, 64, 1, 1, 1, 1),           # L = 1
    (1, 16, 4, 128, 384, 128, 130, 3),   # Lq > one tile of query rows
]


def _run_small(case):
    b, hq, hkv, d, L, B, lq, T = case
    w, x = make(*case)
    m = sa()
    # ---------------- Phase 1
    o, lse = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], B)
    ro, rl = oracle.phase1(to_np(x["q_ctx"]), to_np(x["k_ctx"]), to_np(x["v_ctx"]), B)
    check_rows(to_np(o), ro, to_np(lse), rl, f"phase1 {case}")
    # ---------------- Phase 2: query
    cap = lq + T
    kc = torch.full((b, cap, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))  # rows not yet written hold NaN on purpose
    oq, lq_lse = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"],
                                kc, vc, B)
    rq, rql = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                  to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(oq), rq, to_np(lq_lse), rql, f"query {case}")
    assert torch.equal(kc[:, :lq], x["k_qry"]) and torch.equal(vc[:, :lq], x["v_qry"])
    # ---------------- Phase 2: decode steps
    k_cache = np.zeros((b, cap, hkv, d))
    v_cache = np.zeros((b, cap, hkv, d))
    k_cache[:, :lq] = to_np(x["k_qry"])
    v_cache[:, :lq] = to_np(x["v_qry"])
    for t in range(T):
        od, ld = m.phase2_decode(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"],
                                 x["v_ctx"], kc, vc, lq + t, B)
        ro_d, rl_d, k_cache, v_cache = oracle.phase2_decode(
            to_np(x["q_dec"][t]), to_np(x["k_dec"][t]), to_np(x["v_dec"][t]), to_np(x["k_ctx"]),
            to_np(x["v_ctx"]), k_cache, v_cache, lq + t)
        check_rows(to_np(od), ro_d, to_np(ld), rl_d, f"decode {case} t={t}")
        assert torch.equal(kc[:, lq + t], x["k_dec"][t][:, 0])
    assert m.device_status() == 0


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c)))
def test_small_shapes_all_rows(case):
    _run_small(case)


def test_phase1_deterministic():
    w, x = make(1, 4, 2, 128, 1500, 512, 1, 1, seed=3)
    m = sa()
    o1, l1 = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], 512)
    o2, l2 = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], 512)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("S,d", [(7, 128), (1, 128), (8, 128), (9, 128), (17, 128), (33, 128),
                                 (70, 128), (19, 64), (41, 64)])
def test_lse_merge_kernel_against_oracle(S, d):
    """Split counts on both sides of the kernel's groups of 8 partial rows and its
    32-split LSE chunks, an empty split, and one row every split of which is empty."""
    g = torch.Generator(device="cpu").manual_seed(5 + S)
    b, T, H = 2, 3, 4
    o_parts = torch.randn(S, b, T, H, d, generator=g)
    lse_parts = torch.randn(S, b, H, T, generator=g) * 3
    if S > 1:
        lse_parts[S // 2] = float("-inf")  # an empty split
    lse_parts[:, 1, 2, 0] = float("-inf")  # a row that no split saw
    o, lse = sa().lse_merge(o_parts.cuda(), lse_parts.cuda())
    ro, rl = oracle.lse_merge(o_parts.numpy().transpose(0, 1, 3, 2, 4),
                              lse_parts.numpy())  # oracle wants [S, b, H, T, d]
    og, lg = to_np(o).transpose(0, 2, 1, 3), to_np(lse).copy()
    # the empty row: lse -inf and a zero output on both sides
    assert np.isneginf(lg[1, 2, 0]) and np.isneginf(rl[1, 2, 0]) and not og[1, 2, 0].any()
    rl = rl.copy()
    lg[1, 2, 0] = rl[1, 2, 0] = 0.0
    check_rows(og, ro, lg, rl, "merge")


def test_simple_kernels_agree_with_oracle():
    w, x = make(1, 4, 2, 64, 600, 200, 4, 1, seed=7)
    m = sa()
    o, l = m.simple_phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], 200)
    ro, rl = oracle.phase1(to_np(x["q_ctx"]), to_np(x["k_ctx"]), to_np(x["v_ctx"]), 200)
    check_rows(to_np(o), ro, to_np(l), rl, "simple phase1")
    cap = 8
    kc = torch.zeros((1, cap, 2, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[:, :4], vc[:, :4] = x["k_qry"], x["v_qry"]
    o, l = m.simple_phase2(x["q_qry"], x["k_ctx"], x["v_ctx"], kc, vc, 200, 0, True)
    rq, rql = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                  to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(o), rq, to_np(l), rql, "simple phase2")


def test_fma_pipe_exp2_accuracy():
    """The softmax's FMA-pipe 2^x against float64 2^x (and CUDA's own exp2f for
    reference): relative error within the fitted 7.5e-5 bound where the result
    is a normal float (x > -125); near 2^-126 it is only absolutely tiny."""
    x = torch.cat([torch.linspace(-126.0, 8.0, 1_000_001), torch.tensor([0.0, -0.5, 0.5, 7.999])])
    y = sa().selftest_exp2(x.cuda()).cpu().double()
    ref = torch.exp2(x.double())
    normal = x > -125.0
    rel = ((y - ref).abs() / ref)[normal].max().item()
    assert rel < 7.6e-5, rel
    ref32 = torch.exp2(x.cuda()).cpu().double()
    assert ((y - ref32).abs() / ref32)[normal].max().item() < 7.7e-5
    assert (y - ref)[~normal].abs().max().item() < 2.0 ** -135
    # below the range the result is a tiny non-negative float, never NaN
    lo = sa().selftest_exp2(torch.tensor([-127.0, -1e4, float("-inf")], device="cuda")).cpu()
    assert torch.isfinite(lo).all() and (lo >= 0).all() and (lo < 1.2e-38).all()


@pytest.mark.parametrize("nbytes,ctas", [(16, 1), (32768 * 5 + 48, 2), (32768 * 37, 3),
                                         (32768 * 64 - 16, 148)])
def test_read_probe_reads_every_chunk(nbytes, ctas):
    """The read-only bandwidth probe visits every 32 KB chunk (block b takes chunks
    b, b + ctas, ...; a short last chunk included): each block's XOR of its
    chunks' first words matches the host's."""
    g = torch.Generator().manual_seed(nbytes)
    words = torch.randint(0, 2 ** 31 - 1, (nbytes // 4,), generator=g, dtype=torch.int32)
    sink = torch.full((ctas,), -1, dtype=torch.int32, device="cuda")
    sa().selftest_read(words.cuda(), sink, ctas)
    assert sa().device_status() == 0
    first = words[::32768 // 4].numpy()  # first word of every chunk
    want = [int(np.bitwise_xor.reduce(first[b::ctas])) if b < len(first) else 0
            for b in range(ctas)]
    assert sink.cpu().numpy().tolist() == want


def test_wait_timeout_is_reported_not_trapped():
    m = sa()
    assert m.device_status() == 0
    m.selftest_wait_timeout(20_000_000)  # 20 ms
    assert m.device_status() == 6        # STAR_ERR_TIMEOUT, then cleared
    assert m.device_status() == 0
    # the context is still usable
    t = torch.ones(4, device="cuda")
    assert float(t.sum()) == 4.0


# ------------------------------------------------------------------ full-size workloads
def _sample_rows(w, rng, extra=()):
    L, B = w.ctx_len, w.block_size
    rows = set(extra)
    for start, end in oracle.block_plan(L, B):
        for t in (start, start + 1, start + 127, start + 128, end - 129, end - 128, end - 1):
            if start <= t < end:
                rows.add(t)
    rows.update(int(t) for t in rng.integers(0, L, size=96))
    return np.array(sorted(rows))


def _phase1_sampled(w, x, o, lse, heads):
    rng = np.random.default_rng(11)
    plants = [p for p in workloads.plan_plants(w) if p.q_where == "ctx"]
    for bb in range(w.batch):
        for h in heads:
            g = oracle.kv_head_of(h, w.num_q_heads, w.num_kv_heads)
            extra = [p.q_token for p in plants if p.batch == bb and p.q_head == h]
            rows = _sample_rows(w, rng, extra)
            q = x["q_ctx"][bb, :, h].float().cpu().numpy()
            k = x["k_ctx"][bb, :, g].float().cpu().numpy()
            v = x["v_ctx"][bb, :, g].float().cpu().numpy()
            ro, rl = oracle.phase1_head(q, k, v, w.block_size, w.softmax_scale, rows)
            rows_t = torch.as_tensor(rows, device="cuda")
            check_rows(to_np(o[bb, rows_t, h]), ro, to_np(lse[bb, h, rows_t]), rl,
                       f"{w.name} phase1 b={bb} h={h}")


def _phase2_sampled(w, x, heads, steps):
    m = sa()
    b, hkv, d, lq = w.batch, w.num_kv_heads, w.head_dim, w.query_len
    kc = torch.zeros((b, w.cache_capacity, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    oq, lql = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc,
                             w.block_size)
    kc2, vc2 = kc.clone(), vc.clone()
    ws = m.fused_decode_workspace(b, w.num_q_heads, hkv, d, w.ctx_len, w.block_size, "cuda")
    outs, outs_fused = {}, {}
    for t in range(max(steps) + 1):
        args = (x["q_dec"][t], x["k_dec"][t], x["v_dec"][t], x["k_ctx"], x["v_ctx"])
        outs[t] = m.phase2_decode(*args, kc, vc, lq + t, w.block_size)
        outs_fused[t] = m.phase2_decode_fused(*args, kc2, vc2, lq + t, w.block_size,
                                              workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    for bb in range(b):
        for h in heads:
            g = oracle.kv_head_of(h, w.num_q_heads, hkv)
            kctx = x["k_ctx"][bb, :, g].float().cpu().numpy()
            vctx = x["v_ctx"][bb, :, g].float().cpu().numpy()
            kq = x["k_qry"][bb, :, g].float().cpu().numpy()
            vq = x["v_qry"][bb, :, g].float().cpu().numpy()
            ro, rl = oracle.phase2_query_head(x["q_qry"][bb, :, h].float().cpu().numpy(), kctx,
                                              vctx, kq, vq, w.softmax_scale)
            check_rows(to_np(oq[bb, :, h]), ro, to_np(lql[bb, h]), rl,
                       f"{w.name} query b={bb} h={h}")
            kd = x["k_dec"][:, bb, 0, g].float().cpu().numpy()
            vd = x["v_dec"][:, bb, 0, g].float().cpu().numpy()
            for t in steps:
                ro, rl = oracle.phase2_decode_head(
                    x["q_dec"][t, bb, 0, h].float().cpu().numpy(), kctx, vctx,
                    np.concatenate([kq, kd[:t]]), np.concatenate([vq, vd[:t]]), kd[t], vd[t],
                    w.softmax_scale)
                for kind, res in (("split", outs), ("fused", outs_fused)):
                    od, ld = res[t]
                    check_rows(to_np(od[bb, 0, h])[None], ro[None], to_np(ld[bb, h, 0:1]),
                               np.array([rl]), f"{w.name} {kind} decode t={t} b={bb} h={h}")


FULL = ["llama8b-32k", "llama8b-128k", "70b-128k", "1m"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = workloads.get(name)
    x = workloads.make_inputs(w, device="cuda")
    m = sa()
    o, lse = m.phase1(x["q_ctx"], x["k_ctx"], x["v_ctx"], w.block_size)
    torch.cuda.synchronize()
    G = w.group
    plant_heads = sorted({p.q_head for p in workloads.plan_plants(w)})
    heads = sorted({0, w.num_q_heads - 1, G} | set(plant_heads[:2]))
    _phase1_sampled(w, x, o, lse, heads[:3] if name == "1m" else heads)
    del o, lse
    _phase2_sampled(w, x, heads, steps=[0, 1, w.decode_steps - 1])
    assert m.device_status() == 0


@pytest.mark.parametrize("boost", [20.0, 60.0])
def test_phase1_score_jumps_in_later_tiles(boost):
    """A key whose score towers over everything seen before it, in a late tile of
    its block: a moderate jump (the running max's raise is applied at the next tile)
    and a huge one (the tile is recomputed with its own max). Rows that see the key
    must put nearly all weight on it; all rows match the oracle."""
    m = sa()
    b, hq, hkv, d, L, B = 1, 2, 1, 128, 1536, 768
    w, x = make(b, hq, hkv, d, L, B, 1, 1, seed=12)
    q, k, v = x["q_ctx"].clone(), x["k_ctx"].clone(), x["v_ctx"].clone()
    key = 768 + 500  # block 1, its fourth 128-key tile
    for h in range(hq):
        q[0, key + 10:, h] = q[0, key + 10:, h] * 0 + 1.0 / d ** 0.5
    k[0, key, 0] = boost * torch.ones(d, dtype=torch.bfloat16, device="cuda")  # logit = boost
    o, lse = m.phase1(q, k, v, B)
    ro, rl = oracle.phase1(to_np(q), to_np(k), to_np(v), B)
    check_rows(to_np(o), ro, to_np(lse), rl, f"score jump x{boost}")
    assert m.device_status() == 0


@pytest.mark.parametrize("peak_tile", [0, 3, 6])
def test_query_single_q_tile_combines_two_key_streams(peak_tile):
    """When all query rows fit one 128-row tile, a context split runs the tile twice,
    over the chunk's even and odd K/V tiles, and combines the two softmaxes: a key
    that dominates the row may sit in either stream (tile 3 is odd, 0 and 6 even;
    7 tiles in the chunk, so the odd stream's last step has no keys)."""
    m = sa()
    # 80 blocks of 896 keys: the split plan gives one 7-tile chunk per block
    b, hq, hkv, d, B, lq = 1, 8, 2, 128, 896, 5
    L = 80 * B
    w, x = make(b, hq, hkv, d, L, B, lq, 1, seed=7)
    g = torch.Generator(device="cpu").manual_seed(peak_tile)
    u = torch.randn(d, generator=g)
    u = u / u.norm() * 11.0
    key = peak_tile * 128 + 17
    x["k_ctx"][0, key, 1] = u.to(torch.bfloat16).cuda()
    x["q_qry"][0, 2, 5] = u.to(torch.bfloat16).cuda()  # q-head 5 reads kv-head 1
    kc = torch.zeros((b, lq, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    oq, lse = m.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"], kc, vc, B)
    rq, rl = oracle.phase2_query(to_np(x["q_qry"]), to_np(x["k_qry"]), to_np(x["v_qry"]),
                                 to_np(x["k_ctx"]), to_np(x["v_ctx"]))
    check_rows(to_np(oq), rq, to_np(lse), rl, f"single-tile query, peak in tile {peak_tile}")
    assert float(rl[0, 5, 2]) > 10.0  # the planted key dominates that row
    assert m.device_status() == 0
