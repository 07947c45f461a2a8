"""Seeded synthetic workloads for the Star Attention two-phase hot path.

This module only draws random inputs; it holds none of the attention arithmetic.
Both the CUDA path (through the C-ABI) and the CPU oracle consume what it returns,
so it is the one piece of code they share.

The five workloads restate the shapes the Star Attention pages evaluate on
(Llama-3.1-8B-Instruct attention shapes, 32K..1M-token contexts, block sizes of
1/4..1/32 of the context; "Star Attention: Efficient LLM Inference over Long
Sequences", rebuttal to reviewer EMsM, "Impact of Block Size", and the
abstract). Real model activations are not available, so Q/K/V are drawn
i.i.d. N(0,1)/sqrt(d) in fp32 and rounded to bf16 (round-to-nearest-even).

Planted key/query pairs make softmax peaky on two workloads: a unit direction u
gives q = r*u and k = r*(0.9*u + sqrt(0.19)*w) with w a unit vector orthogonal to
u, and r chosen so that softmax_scale * r^2 * 0.9 = 12 (a logit of about 12
against a background of about 0). Half of the pairs put the query among the
Phase-2 query/decode tokens with the key anywhere in the context; the other half
put the query in a block i>0 and the key in the anchor block b_0 or earlier in
b_i, so that both phases see them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    ctx_len: int
    block_size: int
    query_len: int
    decode_steps: int
    planted_pairs: int = 0
    seed: int = 0

    @property
    def num_blocks(self) -> int:
        return -(-self.ctx_len // self.block_size)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def cache_capacity(self) -> int:
        # query tokens + every decode token, rounded up to a multiple of 64 rows
        need = self.query_len + self.decode_steps
        return -(-need // 64) * 64

    def phase1_flops(self) -> float:
        """Algorithmic Phase-1 FLOPs: unmasked QK^T and PV multiply-adds x2.

        Block 0 is plain causal attention (B(B+1)/2 score pairs per head);
        every other block pairs each of its rows with the whole anchor b_0
        (B columns) plus the causal part of its own block.
        """
        L, B = self.ctx_len, self.block_size
        pairs = 0
        for i in range(self.num_blocks):
            n_i = min(B, L - i * B)
            pairs += n_i * (n_i + 1) // 2
            if i > 0:
                pairs += n_i * B
        return 4.0 * self.head_dim * self.num_q_heads * self.batch * pairs

    def phase1_io_bytes(self) -> int:
        """Bytes Phase 1 must move at least once: Q, K, V read, O and the LSE written."""
        tok = self.batch * self.ctx_len
        return tok * self.head_dim * 2 * (2 * self.num_q_heads + 2 * self.num_kv_heads) + \
            tok * self.num_q_heads * 4

    def query_flops(self) -> float:
        """Algorithmic FLOPs of the Phase-2 query pass: query token j attends to all
        L context keys and to query tokens 0..j (QK^T and PV multiply-adds x2)."""
        lq = self.query_len
        pairs = lq * self.ctx_len + lq * (lq + 1) // 2
        return 4.0 * self.head_dim * self.num_q_heads * self.batch * pairs

    def query_io_bytes(self) -> int:
        """Bytes the query pass must move at least once: the context K/V read, the
        query tokens' Q read, their K/V read and written into the cache, O and the
        LSE written."""
        b, lq, d = self.batch, self.query_len, self.head_dim
        ctx = b * self.ctx_len * self.num_kv_heads * d * 2 * 2
        q = b * lq * self.num_q_heads * d * 2
        kv = b * lq * self.num_kv_heads * d * 2 * 2 * 2
        out = b * lq * self.num_q_heads * (d * 2 + 4)
        return ctx + q + kv + out

    def decode_kv_bytes(self, step: int) -> int:
        """KV bytes a decode step must read once: context + query tokens + decoded
        tokens so far (including the one appended this step), K and V, bf16."""
        keys = self.ctx_len + self.query_len + step + 1
        return self.batch * keys * self.num_kv_heads * self.head_dim * 2 * 2

    def describe(self) -> Dict[str, object]:
        return dataclasses.asdict(self)


WORKLOADS: List[Workload] = [
    Workload("tiny", 1, 2, 2, 64, 2048, 512, 16, 8, 0, 0),
    Workload("llama8b-32k", 1, 32, 8, 128, 32768, 4096, 64, 128, 16, 0),
    Workload("llama8b-128k", 1, 32, 8, 128, 131072, 16384, 128, 256, 0, 0),
    Workload("70b-128k", 2, 64, 8, 128, 131072, 8192, 64, 128, 0, 0),
    Workload("1m", 1, 32, 8, 128, 1048576, 32768, 32, 64, 64, 0),
]
BY_NAME: Dict[str, Workload] = {w.name: w for w in WORKLOADS}


def get(name: str) -> Workload:
    return BY_NAME[name]


# Independent sub-streams, one per tensor, so that drawing one tensor never shifts another.
_STREAMS = {"q_ctx": 1, "k_ctx": 2, "v_ctx": 3, "q_qry": 4, "k_qry": 5, "v_qry": 6,
            "q_dec": 7, "k_dec": 8, "v_dec": 9}


def _randn_bf16(shape, seed: int, stream: str, head_dim: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + _STREAMS[stream])
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(1.0 / math.sqrt(head_dim))
    return x.to(torch.bfloat16)


@dataclasses.dataclass
class Plant:
    """One planted pair: the query row (batch, q-head, where, token) and the key
    (batch, kv-head, where, token). `where` is 'ctx', 'qry' or 'dec'; for 'dec'
    the token index is the decode step."""
    batch: int
    q_head: int
    q_where: str
    q_token: int
    kv_head: int
    k_where: str
    k_token: int


def plan_plants(w: Workload) -> List[Plant]:
    rng = np.random.RandomState(w.seed * 7919 + 17)
    plants: List[Plant] = []
    G = w.group
    n = w.num_blocks
    for p in range(w.planted_pairs):
        b = int(rng.randint(w.batch))
        h = int(rng.randint(w.num_q_heads))
        kvh = h // G
        if p % 2 == 0:
            # Phase-2 pair: query among query/decode tokens, key uniform over the context.
            if rng.rand() < 0.5 or w.decode_steps == 0:
                qw, qt = "qry", int(rng.randint(w.query_len))
            else:
                qw, qt = "dec", int(rng.randint(w.decode_steps))
            plants.append(Plant(b, h, qw, qt, kvh, "ctx", int(rng.randint(w.ctx_len))))
        else:
            # Phase-1 pair: query in a block i>0, key in the anchor or earlier in b_i.
            if n < 2:
                i = 0
            else:
                i = int(rng.randint(1, n))
            lo = i * w.block_size
            hi = min(w.ctx_len, lo + w.block_size)
            qt = int(rng.randint(lo, hi))
            if i > 0 and rng.rand() < 0.5:
                kt = int(rng.randint(0, w.block_size))
            else:
                kt = int(rng.randint(lo, qt + 1))
            plants.append(Plant(b, h, "ctx", qt, kvh, "ctx", kt))
    return plants


def _plant_vectors(w: Workload, rng: np.random.RandomState):
    d = w.head_dim
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    z = rng.standard_normal(d)
    z -= z.dot(u) * u
    z /= np.linalg.norm(z)
    r = math.sqrt(12.0 / (0.9 * w.softmax_scale))
    q = r * u
    k = r * (0.9 * u + math.sqrt(0.19) * z)
    return q, k


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None,
                parts=("ctx", "qry", "dec")) -> Dict[str, torch.Tensor]:
    """Draw the workload's tensors on `device`.

    Returns a dict with (as requested by `parts`):
      q_ctx [b, L, Hq, d], k_ctx / v_ctx [b, L, Hkv, d]
      q_qry [b, Lq, Hq, d], k_qry / v_qry [b, Lq, Hkv, d]
      q_dec [T, b, 1, Hq, d], k_dec / v_dec [T, b, 1, Hkv, d]
    all bf16, contiguous, token-major.
    """
    seed = w.seed if seed is None else seed
    b, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    out: Dict[str, torch.Tensor] = {}
    if "ctx" in parts:
        out["q_ctx"] = _randn_bf16((b, w.ctx_len, Hq, d), seed, "q_ctx", d, device)
        out["k_ctx"] = _randn_bf16((b, w.ctx_len, Hkv, d), seed, "k_ctx", d, device)
        out["v_ctx"] = _randn_bf16((b, w.ctx_len, Hkv, d), seed, "v_ctx", d, device)
    if "qry" in parts:
        out["q_qry"] = _randn_bf16((b, w.query_len, Hq, d), seed, "q_qry", d, device)
        out["k_qry"] = _randn_bf16((b, w.query_len, Hkv, d), seed, "k_qry", d, device)
        out["v_qry"] = _randn_bf16((b, w.query_len, Hkv, d), seed, "v_qry", d, device)
    if "dec" in parts:
        out["q_dec"] = _randn_bf16((w.decode_steps, b, 1, Hq, d), seed, "q_dec", d, device)
        out["k_dec"] = _randn_bf16((w.decode_steps, b, 1, Hkv, d), seed, "k_dec", d, device)
        out["v_dec"] = _randn_bf16((w.decode_steps, b, 1, Hkv, d), seed, "v_dec", d, device)
    if w.planted_pairs:
        rng = np.random.RandomState(seed * 104729 + 3)
        for p in plan_plants(w):
            qv, kv = _plant_vectors(w, rng)
            qt = torch.tensor(qv, dtype=torch.float32).to(torch.bfloat16)
            kt = torch.tensor(kv, dtype=torch.float32).to(torch.bfloat16)
            qkey = {"ctx": "q_ctx", "qry": "q_qry", "dec": "q_dec"}[p.q_where]
            if qkey in out:
                if p.q_where == "dec":
                    out[qkey][p.q_token, p.batch, 0, p.q_head] = qt.to(device)
                else:
                    out[qkey][p.batch, p.q_token, p.q_head] = qt.to(device)
            if "k_ctx" in out:
                out["k_ctx"][p.batch, p.k_token, p.kv_head] = kt.to(device)
    return out


def make_head_slices(w: Workload, rows, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """The one-head slices a bounded CPU timing sample needs, drawn on the host
    with the workload's distribution (N(0,1)/sqrt(d), rounded to bf16) from the
    same per-tensor seeds, without materialising the whole batch x heads tensors:
      q_ctx [L, d] (zero except at `rows`), k_ctx / v_ctx [L, d] (one kv-head),
      q_qry / k_qry / v_qry [Lq, d], q_dec / k_dec / v_dec [d] (the first step),
    as float32 arrays holding bf16 values. Planted pairs are left out (they do not
    change how much work the oracle does). The values are not those of the GPU
    arm's tensors (a host generator and a device generator draw different
    streams); only shapes and distribution match."""
    seed = w.seed if seed is None else seed
    d, L = w.head_dim, w.ctx_len
    rows = np.asarray(rows, dtype=np.int64)
    f = lambda t: t.float().numpy()  # noqa: E731
    q = np.zeros((L, d), dtype=np.float32)
    q[rows] = f(_randn_bf16((len(rows), d), seed, "q_ctx", d, "cpu"))
    out = {"q_ctx": q,
           "k_ctx": f(_randn_bf16((L, d), seed, "k_ctx", d, "cpu")),
           "v_ctx": f(_randn_bf16((L, d), seed, "v_ctx", d, "cpu"))}
    for name in ("q_qry", "k_qry", "v_qry"):
        out[name] = f(_randn_bf16((w.query_len, d), seed, name, d, "cpu"))
    for name in ("q_dec", "k_dec", "v_dec"):
        out[name] = f(_randn_bf16((d,), seed, name, d, "cpu"))
    return out


def l2_flush_bytes() -> int:
    """Size of the buffer written between timed iterations to evict the 126 MB L2."""
    return 256 << 20
