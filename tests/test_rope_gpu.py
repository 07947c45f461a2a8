"""RoPE kernel and the anchor-position variant of Phase 1 against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import check_rows, to_np

pytestmark = pytest.mark.gpu


def sa():
    import block_sparse_attention_phase_b200 as m
    return m


def raw(b, L, h, d, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(b, L, h, d, generator=g).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("d,pos0", [(128, 0), (64, 1_000_003)])
def test_rope_matches_oracle(d, pos0):
    m = sa()
    b, L, hq, hkv, B = 2, 300, 4, 2, 128
    q, k = raw(b, L, hq, d, 1), raw(b, L, hkv, d, 2)
    inv = m.rope_inv_freq(d)
    qr, kr, qa = m.rope(q, k, inv, pos0=pos0, block_size=B, want_anchor=True)
    pos = pos0 + np.arange(L)
    ref_q = oracle.rope(to_np(q), pos, inv)
    ref_k = oracle.rope(to_np(k), pos, inv)
    # one bf16 rounding of a value computed in fp32 from exact bf16 inputs
    for got, ref in ((qr, ref_q), (kr, ref_k)):
        err = np.abs(to_np(got) - ref)
        assert (err <= 2.0 ** -8 * np.abs(ref) + 1e-6).all(), err.max()
    blk = np.arange(L) // B
    apos = pos0 + np.arange(L) - np.where(blk > 0, (blk - 1) * B, 0)
    ref_a = oracle.rope(to_np(q), apos, inv)
    err = np.abs(to_np(qa) - ref_a)
    assert (err <= 2.0 ** -8 * np.abs(ref_a) + 1e-6).all(), err.max()
    # in place gives the same bytes
    q2, k2 = q.clone(), k.clone()
    m.rope(q2, k2, inv, pos0=pos0, block_size=B, inplace=True)
    assert torch.equal(q2, qr) and torch.equal(k2, kr)


@pytest.mark.parametrize("variant", ["original", "adjacent"])
def test_phase1_with_rope_anchor_positions(variant):
    m = sa()
    b, L, hq, hkv, d, B = 1, 1500, 4, 2, 128, 512
    q, k = raw(b, L, hq, d, 3), raw(b, L, hkv, d, 4)
    v = (raw(b, L, hkv, d, 5).float() / d ** 0.5).to(torch.bfloat16)
    inv = m.rope_inv_freq(d, base=10000.0)
    qr, kr, qa = m.rope(q, k, inv, block_size=B, want_anchor=True)
    if variant == "original":
        o, lse = m.phase1(qr, kr, v, B)
    else:
        o, lse = m.phase1_anchor_q(qr, qa, kr, v, B)
    ro, rl = oracle.phase1_rope(to_np(q), to_np(k), to_np(v), B, inv, variant)
    check_rows(to_np(o), ro, None, None, f"rope phase1 {variant}")
    # The GPU path stores the rotated q and k in bf16 (at most 2^-9 relative per
    # element, norms kept by the rotation); the oracle rotates exactly. A score
    # then moves by at most scale * 2^-8 * |q_t| * max_j |k_j|, and the LSE by at
    # most the largest such move over the row's keys.
    scale = 1.0 / d ** 0.5
    qn = np.linalg.norm(to_np(q), axis=-1)                  # [b, L, Hq]
    kmax = np.linalg.norm(to_np(k), axis=-1).max(axis=1)     # [b, Hkv]
    bound = scale * 2.0 ** -8 * qn * np.repeat(kmax, hq // hkv, axis=1)[:, None, :]
    lerr = np.abs(to_np(lse) - rl)                           # [b, Hq, L]
    assert (lerr <= bound.transpose(0, 2, 1) + 1e-3).all(), float((lerr - bound.transpose(0, 2, 1)).max())
    if variant == "adjacent":
        # blocks 0 and 1 are the same in both variants (bit for bit: same tiles)
        o2, l2 = m.phase1(qr, kr, v, B)
        assert torch.equal(o[:, :2 * B], o2[:, :2 * B])
        assert not torch.equal(o[:, 2 * B:], o2[:, 2 * B:])
    assert m.device_status() == 0


@pytest.mark.parametrize("variant", ["original", "adjacent"])
def test_model_stack_matches_oracle(variant):
    """Two layers: context, query tokens and decode steps through projections, RoPE,
    Phase 1 and Phase 2 against the float64 model. Every tensor between layers is
    bf16 on the GPU (projections, rotated q/k, attention outputs, residual), so the
    tolerance is relative to the hidden states' size: a few bf16 roundings per layer."""
    from block_sparse_attention_phase_b200.model import StarModel
    b, L, hidden, hq, hkv, d, B, Lq, T = 1, 1100, 256, 4, 2, 64, 256, 5, 3
    mdl = StarModel(2, hidden, hq, hkv, d, B, b, L, Lq + T, rope_base=10000.0,
                    anchor_positions=variant, seed=7)
    g = torch.Generator(device="cpu").manual_seed(8)
    x_ctx = torch.randn(b, L, hidden, generator=g).to(torch.bfloat16).cuda()
    x_q = torch.randn(b, Lq, hidden, generator=g).to(torch.bfloat16).cuda()
    x_d = [torch.randn(b, 1, hidden, generator=g).to(torch.bfloat16).cuda() for _ in range(T)]
    y_ctx = mdl.prefill(x_ctx)
    y_q = mdl.query(x_q)
    y_d = [mdl.decode(t) for t in x_d]
    r_ctx, r_q, r_d = oracle.model_forward(
        to_np(x_ctx), to_np(x_q), [to_np(t) for t in x_d], [to_np(w) for w in mdl.w_qkv],
        [to_np(w) for w in mdl.w_o], hq, hkv, d, B, mdl.inv_freq, variant)
    for got, ref, what in [(y_ctx, r_ctx, "ctx"), (y_q, r_q, "query")] + \
            [(y, r, f"decode {t}") for t, (y, r) in enumerate(zip(y_d, r_d))]:
        err = np.abs(to_np(got) - ref)
        scale = np.abs(ref).mean()
        assert err.max() <= 0.05 * np.abs(ref).max(), (what, err.max(), np.abs(ref).max())
        assert err.mean() <= 0.01 * scale, (what, err.mean(), scale)
    assert sa().device_status() == 0
