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
