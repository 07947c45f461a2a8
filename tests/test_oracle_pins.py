"""Pins for the CPU oracle: each check ties it to something other than itself.

* torch's scaled_dot_product_attention and logsumexp (library routines) for the
  cases where Star Attention reduces to textbook attention: one block (B >= L)
  and two blocks (the anchor is then the whole preceding context), the first
  and the last row of a block, and exact global attention in Phase 2;
* hand-written key sets (tests/golden) read back through a closed form:
  with q = 0 every visible key gets the same weight, so with one-hot values the
  output row is 1/|K(t)| on exactly the visible positions and lse = ln |K(t)|;
* closed forms: one key gives o = v, lse = s; N identical keys give
  o = mean(v), lse = s + ln N;
* invariants the pages fix: block i does not read blocks other than b_0 and
  b_i; the LSE merge is exact and independent of split count and order.

The last test plants plausible mistakes in the oracle (on the CPU) and checks
that at least one pin catches each of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import star_oracle as so

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers
def sdpa_rows(q, k, v, scale, mask=None):
    """torch SDPA (float64, CPU) of rows q [R,d] over keys k, v [N,d]; mask [R,N] bool."""
    qt = torch.tensor(q, dtype=torch.float64)[None, None]
    kt = torch.tensor(k, dtype=torch.float64)[None, None]
    vt = torch.tensor(v, dtype=torch.float64)[None, None]
    m = None if mask is None else torch.tensor(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    s = scale * (torch.tensor(q) @ torch.tensor(k).T)
    if mask is not None:
        s = s.masked_fill(~torch.tensor(mask), float("-inf"))
    return o[0, 0].numpy(), torch.logsumexp(s, dim=1).numpy()


def sdpa_causal_gqa(q, k, v, scale):
    """Plain causal attention for q [L,Hq,d], k, v [L,Hkv,d] via torch SDPA."""
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    qt = torch.tensor(q).permute(1, 0, 2)
    kt = torch.tensor(k).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.tensor(v).permute(1, 0, 2).repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    L = q.shape[0]
    s = scale * qt @ kt.transpose(1, 2)
    s = s.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    return o.permute(1, 0, 2).numpy(), torch.logsumexp(s, dim=2).numpy()  # [L,Hq,d], [Hq,L]


def rand(rng, *shape):
    return rng.standard_normal(shape)


def read_cases(name):
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case"):
                cur = {"args": [int(x) for x in line.split()[1:]], "rows": {}}
                cases.append(cur)
            else:
                key, vals = line.split(":")
                cur["rows"][key.strip()] = vals.split()
    return cases


# ----------------------------------------------------------------- pin checks
# Each check raises AssertionError on a mismatch; the mutation test reuses them.

def check_single_block_is_causal(seed=0):
    rng = np.random.default_rng(seed)
    for L, B in [(37, 37), (37, 64), (1, 1), (12, 100)]:
        q, k, v = rand(rng, 1, L, 4, 16), rand(rng, 1, L, 2, 16), rand(rng, 1, L, 2, 16)
        o, lse = oracle.phase1(q, k, v, B)
        ro, rl = sdpa_causal_gqa(q[0], k[0], v[0], 0.25)
        np.testing.assert_allclose(o[0], ro, atol=1e-12, rtol=1e-10)
        np.testing.assert_allclose(lse[0], rl, atol=1e-12, rtol=1e-10)


def check_two_blocks_is_full_causal(seed=1):
    rng = np.random.default_rng(seed)
    for L, B in [(40, 20), (37, 20), (33, 32)]:
        q, k, v = rand(rng, 1, L, 4, 8), rand(rng, 1, L, 1, 8), rand(rng, 1, L, 1, 8)
        o, lse = oracle.phase1(q, k, v, B, scale=0.3)
        ro, rl = sdpa_causal_gqa(q[0], k[0], v[0], 0.3)
        np.testing.assert_allclose(o[0], ro, atol=1e-12, rtol=1e-10)
        np.testing.assert_allclose(lse[0], rl, atol=1e-12, rtol=1e-10)


def check_phase1_keysets_golden():
    for case in read_cases("phase1_keysets.txt"):
        L, B = case["args"]
        d = L  # one-hot values need d >= L
        q = np.zeros((1, L, 1, d))
        k = np.random.default_rng(L * 31 + B).standard_normal((1, L, 1, d))
        v = np.eye(L)[None, :, None, :]
        o, lse = oracle.phase1(q, k, v, B)
        for t in range(L):
            vis = [int(x) for x in case["rows"][str(t)]]
            want = np.zeros(L)
            want[vis] = 1.0 / len(vis)
            np.testing.assert_allclose(o[0, t, 0], want, atol=1e-14)
            assert abs(lse[0, 0, t] - math.log(len(vis))) < 1e-12


def check_first_and_last_row_of_block(seed=2):
    rng = np.random.default_rng(seed)
    L, B, d = 50, 12, 8
    q, k, v = rand(rng, 1, L, 2, d), rand(rng, 1, L, 2, d), rand(rng, 1, L, 2, d)
    o, lse = oracle.phase1(q, k, v, B)
    for start, end in [(12, 24), (24, 36), (48, 50)]:
        for h in range(2):
            # first row of the block: the anchor b_0 and itself
            keys = list(range(B)) + [start]
            ro, rl = sdpa_rows(q[0, [start], h], k[0, keys, h], v[0, keys, h], 1 / math.sqrt(d))
            np.testing.assert_allclose(o[0, start, h], ro[0], atol=1e-12)
            assert abs(lse[0, h, start] - rl[0]) < 1e-12
            # last row: the whole anchor and the whole block, no mask
            keys = list(range(B)) + list(range(start, end))
            ro, rl = sdpa_rows(q[0, [end - 1], h], k[0, keys, h], v[0, keys, h], 1 / math.sqrt(d))
            np.testing.assert_allclose(o[0, end - 1, h], ro[0], atol=1e-12)
            assert abs(lse[0, h, end - 1] - rl[0]) < 1e-12


def check_block_independence(seed=3):
    rng = np.random.default_rng(seed)
    L, B, d = 64, 16, 8
    q, k, v = rand(rng, 1, L, 2, d), rand(rng, 1, L, 1, d), rand(rng, 1, L, 1, d)
    o, _ = oracle.phase1(q, k, v, B)
    i = 3  # rows 48..63
    for j in (1, 2):  # any block other than b_0 and b_i
        k2, v2 = k.copy(), v.copy()
        k2[:, j * B:(j + 1) * B] += rand(rng, 1, B, 1, d)
        v2[:, j * B:(j + 1) * B] += rand(rng, 1, B, 1, d)
        o2, _ = oracle.phase1(q, k2, v2, B)
        np.testing.assert_array_equal(o2[:, i * B:], o[:, i * B:])
    k3 = k.copy()
    k3[:, :B] += rand(rng, 1, B, 1, d)  # the anchor does matter
    o3, _ = oracle.phase1(q, k3, v, B)
    assert np.abs(o3[:, i * B:] - o[:, i * B:]).max() > 1e-3


def check_gqa_mapping(seed=4):
    rng = np.random.default_rng(seed)
    L, B, d, Hq, Hkv = 20, 8, 4, 6, 2
    q, k, v = rand(rng, 1, L, Hq, d), rand(rng, 1, L, Hkv, d), rand(rng, 1, L, Hkv, d)
    o, _ = oracle.phase1(q, k, v, B)
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G  # contiguous grouping: heads 0..G-1 share kv-head 0
        oh, _ = oracle.phase1(q[:, :, [h]], k[:, :, [g]], v[:, :, [g]], B)
        np.testing.assert_array_equal(o[:, :, h], oh[:, :, 0])


def check_closed_forms():
    rng = np.random.default_rng(5)
    d = 16
    q, k, v = rand(rng, 1, d), rand(rng, 1, d), rand(rng, 1, d)
    o, lse = oracle.attend(q, k, v, 0.7)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)
    assert abs(lse[0] - 0.7 * float(q[0] @ k[0])) < 1e-12
    N = 9
    kk = np.repeat(k, N, axis=0)
    vv = rand(rng, N, d)
    o, lse = oracle.attend(q, kk, vv, 0.7)
    np.testing.assert_allclose(o[0], vv.mean(axis=0), atol=1e-14)
    assert abs(lse[0] - (0.7 * float(q[0] @ k[0]) + math.log(N))) < 1e-12
    # one query row with no visible key
    o, lse = oracle.attend(q, kk, vv, 0.7, np.zeros((1, N), dtype=bool))
    assert np.all(o == 0) and lse[0] == -np.inf


def check_phase2_query_is_global(seed=6):
    rng = np.random.default_rng(seed)
    L, B, Lq, d = 45, 10, 7, 8
    q = rand(rng, Lq, d)
    kc, vc, kq, vq = rand(rng, L, d), rand(rng, L, d), rand(rng, Lq, d), rand(rng, Lq, d)
    keys = np.concatenate([kc, kq])
    vals = np.concatenate([vc, vq])
    mask = np.concatenate([np.ones((Lq, L), bool), np.tril(np.ones((Lq, Lq), bool))], axis=1)
    ro, rl = sdpa_rows(q, keys, vals, 0.35, mask)
    for fn in (lambda: oracle.phase2_query_head(q, kc, vc, kq, vq, 0.35),
               lambda: oracle.phase2_query_head_blockwise(q, kc, vc, kq, vq, B, 0.35)):
        o, lse = fn()
        np.testing.assert_allclose(o, ro, atol=1e-12)
        np.testing.assert_allclose(lse, rl, atol=1e-12)


def check_phase2_keysets_golden():
    for case in read_cases("phase2_keysets.txt"):
        L, Lq, T = case["args"]
        n_keys = L + Lq + T
        d = n_keys
        kc = np.random.default_rng(1).standard_normal((L, d))
        kq = np.random.default_rng(2).standard_normal((Lq, d))
        kd = np.random.default_rng(3).standard_normal((T, d))
        eye = np.eye(n_keys)
        vc, vq, vd = eye[:L], eye[L:L + Lq], eye[L + Lq:]

        def pos(name):
            return int(name[1:]) if name[0] == "c" else L + int(name[1:])

        o, lse = oracle.phase2_query_head(np.zeros((Lq, d)), kc, vc, kq, vq, 1.0)
        for j in range(Lq):
            vis = [pos(x) for x in case["rows"][f"q{j}"]]
            want = np.zeros(n_keys)
            want[vis] = 1.0 / len(vis)
            np.testing.assert_allclose(o[j], want, atol=1e-14)
            assert abs(lse[j] - math.log(len(vis))) < 1e-12
        kcache, vcache = kq, vq
        for t in range(T):
            o, lse = oracle.phase2_decode_head(np.zeros(d), kc, vc, kcache, vcache, kd[t], vd[t], 1.0)
            vis = [pos(x) for x in case["rows"][f"d{t}"]]
            want = np.zeros(n_keys)
            want[vis] = 1.0 / len(vis)
            np.testing.assert_allclose(o, want, atol=1e-14)
            assert abs(lse - math.log(len(vis))) < 1e-12
            kcache = np.concatenate([kcache, kd[t][None]])
            vcache = np.concatenate([vcache, vd[t][None]])


def check_merge_split_invariance(seed=7):
    rng = np.random.default_rng(seed)
    N, d, R = 40, 6, 3
    q, k, v = rand(rng, R, d), rand(rng, N, d), rand(rng, N, d)
    ro, rl = sdpa_rows(q, k, v, 0.5)
    for _ in range(5):
        cuts = np.sort(rng.choice(np.arange(1, N), size=int(rng.integers(1, 8)), replace=False))
        bounds = [0] + list(cuts) + [N]
        parts = [oracle.attend(q, k[a:b], v[a:b], 0.5) for a, b in zip(bounds[:-1], bounds[1:])]
        order = rng.permutation(len(parts))
        parts = [parts[i] for i in order]
        # an empty partial (no visible key) must weigh nothing
        parts.append((np.zeros((R, d)), np.full(R, -np.inf)))
        o, lse = oracle.lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        np.testing.assert_allclose(o, ro, atol=1e-12)
        np.testing.assert_allclose(lse, rl, atol=1e-12)


def check_decode_matches_query_rows(seed=8):
    rng = np.random.default_rng(seed)
    b, L, Lq, T, Hq, Hkv, d = 1, 30, 4, 3, 4, 2, 8
    kc, vc = rand(rng, b, L, Hkv, d), rand(rng, b, L, Hkv, d)
    qq, kq, vq = rand(rng, b, Lq + T, Hq, d), rand(rng, b, Lq + T, Hkv, d), rand(rng, b, Lq + T, Hkv, d)
    full_o, full_lse = oracle.phase2_query(qq, kq, vq, kc, vc)
    cap = Lq + T
    kcache = np.zeros((b, cap, Hkv, d))
    vcache = np.zeros((b, cap, Hkv, d))
    kcache[:, :Lq], vcache[:, :Lq] = kq[:, :Lq], vq[:, :Lq]
    for t in range(T):
        pos = Lq + t
        o, lse, kcache, vcache = oracle.phase2_decode(qq[:, [pos]], kq[:, [pos]], vq[:, [pos]],
                                                      kc, vc, kcache, vcache, pos)
        np.testing.assert_allclose(o[:, 0], full_o[:, pos], atol=1e-12)
        np.testing.assert_allclose(lse[:, :, 0], full_lse[:, :, pos], atol=1e-12)


def check_phase1_varlen_per_sequence(seed=9):
    """Varlen Phase 1 = each packed sequence on its own. Every sequence here has at
    most two blocks, so its Phase 1 is plain causal attention (torch SDPA)."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, d = 8, 4, 2, 16
    lens = [5, 0, 16, 11, 1, 8]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    total = int(cu[-1])
    q, k, v = rand(rng, total, Hq, d), rand(rng, total, Hkv, d), rand(rng, total, Hkv, d)
    scale = 0.3
    o, lse = oracle.phase1_varlen(q, k, v, list(cu), B, scale)
    assert o.shape == (total, Hq, d) and lse.shape == (Hq, total)
    for a, e in zip(cu[:-1], cu[1:]):
        if e == a:
            continue
        ro, rl = sdpa_causal_gqa(q[a:e], k[a:e], v[a:e], scale)
        np.testing.assert_allclose(o[a:e], ro, atol=1e-12)
        np.testing.assert_allclose(lse[:, a:e], rl, atol=1e-12)


def check_decode_varlen_is_global_per_sequence(seed=10):
    """Varlen decode: sequence i's new token attends to exactly its own context,
    its own cached rows and itself (torch SDPA over that concatenation), and its
    KV lands at row cache_lens[i] of its own cache only."""
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, cap = 4, 2, 8, 6
    ctx_lens, cache_lens = [7, 0, 12], [2, 5, 0]
    b = len(ctx_lens)
    cu = [0] + list(np.cumsum(ctx_lens))
    kc, vc = rand(rng, cu[-1], Hkv, d), rand(rng, cu[-1], Hkv, d)
    kcache, vcache = rand(rng, b, cap, Hkv, d), rand(rng, b, cap, Hkv, d)
    q, k, v = rand(rng, b, 1, Hq, d), rand(rng, b, 1, Hkv, d), rand(rng, b, 1, Hkv, d)
    scale = 0.4
    o, lse, kn, vn = oracle.phase2_decode_varlen(q, k, v, kc, vc, cu, kcache, vcache, cache_lens,
                                                 scale)
    for i in range(b):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            keys = np.concatenate([kc[cu[i]:cu[i + 1], g], kcache[i, :cache_lens[i], g], k[i, :, g]])
            vals = np.concatenate([vc[cu[i]:cu[i + 1], g], vcache[i, :cache_lens[i], g], v[i, :, g]])
            ro, rl = sdpa_rows(q[i, :, h], keys, vals, scale)
            np.testing.assert_allclose(o[i, 0, h], ro[0], atol=1e-12)
            np.testing.assert_allclose(lse[i, h, 0], rl[0], atol=1e-12)
        expect_k = kcache[i].copy()
        expect_k[cache_lens[i]] = k[i, 0]
        np.testing.assert_array_equal(kn[i], expect_k)


def check_rope_is_complex_rotation(seed=11):
    """RoPE against its complex form: (x_f + i x_{f+d/2}) * exp(i p theta_f), plus
    identity at position 0 and preserved norms."""
    rng = np.random.default_rng(seed)
    L, H, d = 9, 3, 16
    x = rand(rng, 2, L, H, d)
    pos = rng.integers(0, 100000, size=L)
    inv = 10000.0 ** (-2 * np.arange(d // 2) / d)
    y = oracle.rope(x, pos, inv)
    z = (x[..., : d // 2] + 1j * x[..., d // 2:]) * np.exp(1j * pos[:, None, None] * inv)
    np.testing.assert_allclose(y, np.concatenate([z.real, z.imag], axis=-1), atol=1e-9)
    np.testing.assert_allclose(oracle.rope(x, np.zeros(L), inv), x, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


def check_anchor_positions(seed=12):
    """'original' anchor positions = Phase 1 on rotated q, k; 'adjacent' = plain
    causal attention (SDPA) over [b_0 ; b_i] rotated at positions 0 .. 2B-1, since
    RoPE scores depend only on position differences; both agree on blocks 0 and 1."""
    rng = np.random.default_rng(seed)
    B, L, d = 6, 22, 8
    q, k, v = rand(rng, L, d), rand(rng, L, d), rand(rng, L, d)
    inv = 500.0 ** (-2 * np.arange(d // 2) / d)
    scale = 0.35
    oo, lo = oracle.phase1_rope_head(q, k, v, B, scale, inv, "original")
    qr = oracle.rope(q[:, None], np.arange(L), inv)[:, 0]
    kr = oracle.rope(k[:, None], np.arange(L), inv)[:, 0]
    ro, rl = oracle.phase1_head(qr, kr, v, B, scale)
    np.testing.assert_allclose(oo, ro, atol=1e-12)
    np.testing.assert_allclose(lo, rl, atol=1e-12)
    oa, la = oracle.phase1_rope_head(q, k, v, B, scale, inv, "adjacent")
    np.testing.assert_allclose(oa[:2 * B], oo[:2 * B], atol=1e-12)
    for start, end in oracle.block_plan(L, B)[1:]:
        seq = np.concatenate([np.arange(B), np.arange(start, end)])
        qs = oracle.rope(q[seq][:, None], np.arange(len(seq)), inv)[:, 0]
        ks = oracle.rope(k[seq][:, None], np.arange(len(seq)), inv)[:, 0]
        n = len(seq)
        so_, sl_ = sdpa_rows(qs, ks, v[seq], scale, np.tril(np.ones((n, n), dtype=bool)))
        np.testing.assert_allclose(oa[start:end], so_[B:], atol=1e-9)
        np.testing.assert_allclose(la[start:end], sl_[B:], atol=1e-9)
    assert np.abs(oa[2 * B:] - oo[2 * B:]).max() > 1e-6  # the variant does change later blocks


def check_model_decode_equals_query(seed=13):
    """In the layer stack, T decode steps after Lq query tokens give the same hidden
    states as Lq + T query tokens (a decoded token sees exactly what a query token
    at its position sees), layer after layer; and 'original' anchors in the stack's
    Phase 1 equal Phase 1 on the rotated q, k."""
    rng = np.random.default_rng(seed)
    b, L, hidden, Hq, Hkv, d, B, Lq, T = 1, 13, 16, 4, 2, 4, 5, 2, 3
    w_qkv = [rand(rng, hidden, (Hq + 2 * Hkv) * d) / 4 for _ in range(2)]
    w_o = [rand(rng, Hq * d, hidden) / 4 for _ in range(2)]
    inv = 100.0 ** (-2 * np.arange(d // 2) / d)
    xc, xq = rand(rng, b, L, hidden), rand(rng, b, Lq, hidden)
    xd = [rand(rng, b, 1, hidden) for _ in range(T)]
    yc, yq, yd = oracle.model_forward(xc, xq, xd, w_qkv, w_o, Hq, Hkv, d, B, inv)
    yc2, yq2, _ = oracle.model_forward(xc, np.concatenate([xq] + xd, axis=1), [], w_qkv, w_o,
                                       Hq, Hkv, d, B, inv)
    np.testing.assert_allclose(yc, yc2, atol=1e-12)
    np.testing.assert_allclose(yq, yq2[:, :Lq], atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(yd[t][:, 0], yq2[:, Lq + t], atol=1e-12)
    # first layer's Phase 1 by hand: rotate, then plain Phase 1
    h = np.asarray(xc) @ w_qkv[0]
    q = h[..., :Hq * d].reshape(b, L, Hq, d)
    k = h[..., Hq * d:(Hq + Hkv) * d].reshape(b, L, Hkv, d)
    v = h[..., (Hq + Hkv) * d:].reshape(b, L, Hkv, d)
    o, _ = oracle.phase1(oracle.rope(q, np.arange(L), inv), oracle.rope(k, np.arange(L), inv), v, B)
    y1, _, _ = oracle.model_forward(xc, xq, [], w_qkv[:1], w_o[:1], Hq, Hkv, d, B, inv)
    np.testing.assert_allclose(y1, xc + o.reshape(b, L, Hq * d) @ w_o[0], atol=1e-12)


def check_query_varlen_is_global_per_sequence(seed=14):
    """Varlen query pass: query token j of sequence i sees exactly its own context
    and its own query tokens 0..j (torch SDPA with that mask)."""
    rng = np.random.default_rng(seed)
    Hq, Hkv, d = 4, 2, 8
    ctx_lens, q_lens = [9, 0, 14], [3, 2, 0]
    cu_c = [0] + list(np.cumsum(ctx_lens))
    cu_q = [0] + list(np.cumsum(q_lens))
    kc, vc = rand(rng, cu_c[-1], Hkv, d), rand(rng, cu_c[-1], Hkv, d)
    q, k, v = rand(rng, cu_q[-1], Hq, d), rand(rng, cu_q[-1], Hkv, d), rand(rng, cu_q[-1], Hkv, d)
    scale = 0.45
    o, lse = oracle.phase2_query_varlen(q, k, v, kc, vc, cu_c, cu_q, scale)
    for i in range(3):
        a, e, c0, c1 = cu_q[i], cu_q[i + 1], cu_c[i], cu_c[i + 1]
        n = e - a
        if n == 0:
            continue
        for h in range(Hq):
            g = h // (Hq // Hkv)
            keys = np.concatenate([kc[c0:c1, g], k[a:e, g]])
            vals = np.concatenate([vc[c0:c1, g], v[a:e, g]])
            mask = np.concatenate([np.ones((n, c1 - c0), dtype=bool),
                                   np.tril(np.ones((n, n), dtype=bool))], axis=1)
            ro, rl = sdpa_rows(q[a:e, h], keys, vals, scale, mask)
            np.testing.assert_allclose(o[a:e, h], ro, atol=1e-12)
            np.testing.assert_allclose(lse[h, a:e], rl, atol=1e-12)


def check_host_partials_merge_to_global(seed=15):
    """The multi-host form of Phase 2: the context cut into per-host runs, each host's
    partial over its own keys (the last one also over the query-local cache), merged
    with the LSE combine, equals the single-host query pass and decode step."""
    rng = np.random.default_rng(seed)
    b, L, Lq, Hq, Hkv, d, cap = 2, 23, 3, 4, 2, 8, 6
    kc, vc = rand(rng, b, L, Hkv, d), rand(rng, b, L, Hkv, d)
    q, k, v = rand(rng, b, Lq, Hq, d), rand(rng, b, Lq, Hkv, d), rand(rng, b, Lq, Hkv, d)
    cuts = [0, 5, 6, 17, L]
    ref_o, ref_l = oracle.phase2_query(q, k, v, kc, vc)
    parts = []
    kcache = vcache = None
    for i, (a, e) in enumerate(zip(cuts[:-1], cuts[1:])):
        host = i == len(cuts) - 2
        o, l, k2, v2 = oracle.phase2_partial(
            q, kc[:, a:e], vc[:, a:e], k if host else None, v if host else None,
            np.zeros((b, cap, Hkv, d)) if host else None, np.zeros((b, cap, Hkv, d)) if host else None, 0)
        if host:
            kcache, vcache = k2, v2
        parts.append((o, l))
    mo, ml = oracle.lse_merge(np.stack([p[0].transpose(0, 2, 1, 3) for p in parts]),
                              np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(mo.transpose(0, 2, 1, 3), ref_o, atol=1e-12)
    np.testing.assert_allclose(ml, ref_l, atol=1e-12)
    # a decode step on top: the new row appended at row Lq of the host's cache
    qd, kd, vd = rand(rng, b, 1, Hq, d), rand(rng, b, 1, Hkv, d), rand(rng, b, 1, Hkv, d)
    rdo, rdl, _, _ = oracle.phase2_decode(qd, kd, vd, kc, vc, kcache, vcache, Lq)
    parts = []
    for i, (a, e) in enumerate(zip(cuts[:-1], cuts[1:])):
        host = i == len(cuts) - 2
        o, l, _, _ = oracle.phase2_partial(qd, kc[:, a:e], vc[:, a:e], kd if host else None,
                                           vd if host else None, kcache if host else None,
                                           vcache if host else None, Lq)
        parts.append((o, l))
    mo, ml = oracle.lse_merge(np.stack([p[0].transpose(0, 2, 1, 3) for p in parts]),
                              np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(mo.transpose(0, 2, 1, 3), rdo, atol=1e-12)
    np.testing.assert_allclose(ml, rdl, atol=1e-12)


ALL_CHECKS = [check_single_block_is_causal, check_two_blocks_is_full_causal,
              check_phase1_keysets_golden, check_first_and_last_row_of_block,
              check_block_independence, check_gqa_mapping, check_closed_forms,
              check_phase2_query_is_global, check_phase2_keysets_golden,
              check_merge_split_invariance, check_decode_matches_query_rows,
              check_phase1_varlen_per_sequence, check_decode_varlen_is_global_per_sequence,
              check_rope_is_complex_rotation, check_anchor_positions,
              check_model_decode_equals_query, check_query_varlen_is_global_per_sequence,
              check_host_partials_merge_to_global]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


def test_default_scale_and_plan():
    assert oracle.default_scale(128) == 1 / math.sqrt(128)
    assert oracle.block_plan(10, 3) == [(0, 3), (3, 6), (6, 9), (9, 10)]
    assert oracle.block_plan(5, 8) == [(0, 5)]
    assert oracle.kv_head_of(5, 32, 8) == 1 and oracle.kv_head_of(31, 32, 8) == 7


# ----------------------------------------------------------------- planted mistakes
def _mut_anchor_previous(t, j, B):
    t, j = np.asarray(t), np.asarray(j)
    return (j <= t) & ((j // B == t // B - 1) | (j // B == t // B))


def _mut_no_anchor(t, j, B):
    t, j = np.asarray(t), np.asarray(j)
    return (j <= t) & (j // B == t // B)


def _mut_strict_causal(t, j, B):
    t, j = np.asarray(t), np.asarray(j)
    return (j < t) & ((j < B) | (j // B == t // B))


def _mut_anchor_not_causal(t, j, B):
    t, j = np.asarray(t), np.asarray(j)
    return (j < B) | ((j // B == t // B) & (j <= t))


def _mut_gqa_modulo(h, Hq, Hkv):
    return h % Hkv


_orig_attend = so.attend


def _mut_attend_no_scale(q, k, v, scale, allowed=None):
    return _orig_attend(q, k, v, 1.0, allowed)


def _mut_attend_transposed(q, k, v, scale, allowed=None):
    # values indexed by the wrong operand (k and v swapped)
    return _orig_attend(q, v, k, scale, allowed)


def _mut_merge_unweighted(o_parts, lse_parts):
    o_parts = np.asarray(o_parts)
    lse_parts = np.asarray(lse_parts)
    fin = np.isfinite(lse_parts)
    o = (o_parts * fin[..., None]).sum(0) / fin.sum(0)[..., None]
    return o, np.log(np.exp(lse_parts).sum(0))


def _mut_varlen_one_context(q, k, v, cu_seqlens, block_size, scale=None):
    # the packed batch treated as one long context (blocks and anchor shared)
    o, lse = so.phase1(q[None], k[None], v[None], block_size, scale)
    return o[0], lse[0]


_orig_decode_varlen = so.phase2_decode_varlen


def _mut_decode_varlen_first_len(q_t, k_t, v_t, k_ctx, v_ctx, cu_ctx, k_cache, v_cache,
                                 cache_lens, scale=None):
    # every sequence given the first sequence's cache length
    return _orig_decode_varlen(q_t, k_t, v_t, k_ctx, v_ctx, cu_ctx, k_cache, v_cache,
                               [cache_lens[0]] * len(cache_lens), scale)


_orig_rope = so.rope


def _mut_rope_sign(x, positions, inv_freq):
    # rotation in the wrong direction
    return _orig_rope(x, -np.asarray(positions), inv_freq)


MUTANTS = {
    "rope_wrong_direction": ("rope", _mut_rope_sign),
    "varlen_one_context": ("phase1_varlen", _mut_varlen_one_context),
    "decode_varlen_first_len": ("phase2_decode_varlen", _mut_decode_varlen_first_len),
    "anchor_is_previous_block": ("phase1_visible", _mut_anchor_previous),
    "no_anchor": ("phase1_visible", _mut_no_anchor),
    "strict_causal": ("phase1_visible", _mut_strict_causal),
    "anchor_sees_future_in_b0": ("phase1_visible", _mut_anchor_not_causal),
    "gqa_modulo": ("kv_head_of", _mut_gqa_modulo),
    "dropped_scale": ("attend", _mut_attend_no_scale),
    "k_v_swapped": ("attend", _mut_attend_transposed),
    "merge_unweighted": ("lse_merge", _mut_merge_unweighted),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(so, attr, fn)
    monkeypatch.setattr(oracle, attr, fn)
    failed = []
    for check in ALL_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
