"""CPU oracle for the Star Attention two-phase hot path (test infrastructure).

This package is the parity reference for the CUDA path. Only the tests,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may import it;
the product path never does. It shares no code with the CUDA library.

Everything here is plain numpy in float64, written from the method's
definition on the Star Attention pages:

* Phase 1 ("Star Attention: Efficient LLM Inference over Long Sequences",
  hotaipapers.com page, podcast section on Phase 1; rebuttal to reviewers EMsM
  and x5MA, "Size of Anchor Block" and "Anchor Block Content and Position"):
  the context is cut into blocks of B tokens; the first block b_0 is placed as
  an anchor in front of every other block b_i, and each block runs causal
  attention over [anchor ; b_i]. Only b_i's own rows are kept.
* Phase 2 (same hotaipapers.com page, Phase 2 paragraph; abstract): the query
  is sent to every block, each block returns its local attention output and one
  scalar (read here as the log-sum-exp), and the query host combines them into
  exact global attention over every cached token, then appends the new token's
  KV to its cache and decodes.

Every function states which of those passages it follows. The pins that tie
the oracle to the pages and to the mathematics live in tests/test_oracle_pins.py.
"""
from .star_oracle import (  # noqa: F401
    default_scale,
    kv_head_of,
    block_plan,
    phase1_visible,
    attend,
    lse_merge,
    phase1_head,
    phase1,
    phase1_varlen,
    phase2_query_head,
    phase2_query_head_blockwise,
    phase2_query,
    phase2_query_varlen,
    phase2_decode_head,
    phase2_decode,
    phase2_decode_varlen,
    phase2_partial,
    rope,
    phase1_rope_head,
    phase1_rope,
    model_forward,
)
