"""A stack of attention layers run the Star Attention way, with random weights.

Each layer projects the hidden states to q, k, v (one bf16 GEMM through cuBLAS,
via torch.matmul: a plain library GEMM), rotates q and k with this library's RoPE
kernel, runs Phase 1 over the context (or Phase 2 for query and decode tokens)
with this library's attention kernels, projects the attention output back with a
second GEMM and adds it to the residual stream. There is no normalisation or MLP:
the stack exists so that Phase 1 and Phase 2 run layer after layer on realistic
inputs (each layer's K/V are the previous layer's outputs, rotated at their
positions), not to model a particular network.

Anchor positions (rebuttal to x5MA, "Anchor Block Content and Position"): with
anchor_positions="original" the anchor tokens keep their own positions 0 .. B-1
in every block's local attention; with "adjacent" they are placed right before
block i, at (i-1)B .. iB-1 (the RoPE kernel then also produces the Q that scores
the anchor tiles, and Phase 1 uses it).
"""
from __future__ import annotations

from typing import List

import torch

from . import StarAttentionLayer, phase1, phase1_anchor_q, rope, rope_inv_freq


class StarModel:
    def __init__(self, num_layers: int, hidden: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, batch: int, ctx_len: int, cache_capacity: int,
                 rope_base: float = 500000.0, anchor_positions: str = "original", device="cuda",
                 seed: int = 0):
        if anchor_positions not in ("original", "adjacent"):
            raise ValueError("anchor_positions must be 'original' or 'adjacent'")
        self.n, self.hidden = num_layers, hidden
        self.hq, self.hkv, self.d = num_q_heads, num_kv_heads, head_dim
        self.B, self.b, self.L = block_size, batch, ctx_len
        self.anchor_positions = anchor_positions
        self.inv_freq = rope_inv_freq(head_dim, rope_base)
        g = torch.Generator(device="cpu").manual_seed(seed)
        qkv_cols = (num_q_heads + 2 * num_kv_heads) * head_dim

        def w(rows, cols):
            return (torch.randn(rows, cols, generator=g) / rows ** 0.5).to(torch.bfloat16).to(device)

        self.w_qkv: List[torch.Tensor] = [w(hidden, qkv_cols) for _ in range(num_layers)]
        self.w_o: List[torch.Tensor] = [w(num_q_heads * head_dim, hidden) for _ in range(num_layers)]
        self.layers = [StarAttentionLayer(batch, num_q_heads, num_kv_heads, head_dim, ctx_len,
                                          block_size, cache_capacity, device=device)
                       for _ in range(num_layers)]
        self.pos = 0  # position of the next token

    def _qkv(self, i: int, x: torch.Tensor):
        b, T, _ = x.shape
        h = torch.matmul(x.reshape(b * T, self.hidden), self.w_qkv[i])
        qd, kd = self.hq * self.d, self.hkv * self.d
        q = h[:, :qd].reshape(b, T, self.hq, self.d).contiguous()
        k = h[:, qd:qd + kd].reshape(b, T, self.hkv, self.d).contiguous()
        v = h[:, qd + kd:].reshape(b, T, self.hkv, self.d).contiguous()
        return q, k, v

    def _out(self, i: int, x: torch.Tensor, o: torch.Tensor) -> torch.Tensor:
        b, T, _ = x.shape
        return x + torch.matmul(o.reshape(b * T, self.hq * self.d), self.w_o[i]).reshape(b, T, -1)

    def prefill(self, x: torch.Tensor) -> torch.Tensor:
        """x [b, L, hidden] bf16: the context through every layer (Phase 1)."""
        adjacent = self.anchor_positions == "adjacent"
        for i in range(self.n):
            q, k, v = self._qkv(i, x)
            q, k, qa = rope(q, k, self.inv_freq, pos0=0, block_size=self.B, want_anchor=adjacent,
                            inplace=True)
            if adjacent:
                o, _ = phase1_anchor_q(q, qa, k, v, self.B, want_lse=False)
            else:
                o, _ = phase1(q, k, v, self.B, want_lse=False)
            # the rotated k and v are this layer's context KV for Phase 2
            layer = self.layers[i]
            layer.k_ctx, layer.v_ctx, layer.cache_len = k, v, 0
            x = self._out(i, x, o)
        self.pos = self.L
        return x

    def query(self, x: torch.Tensor) -> torch.Tensor:
        """x [b, Lq, hidden]: the query tokens (Phase 2), appended to every layer's cache."""
        for i in range(self.n):
            q, k, v = self._qkv(i, x)
            q, k, _ = rope(q, k, self.inv_freq, pos0=self.pos, inplace=True)
            o, _ = self.layers[i].query(q, k, v)
            x = self._out(i, x, o)
        self.pos += x.shape[1]
        return x

    def decode(self, x: torch.Tensor) -> torch.Tensor:
        """x [b, 1, hidden]: one generated token through every layer (Phase 2 decode)."""
        for i in range(self.n):
            q, k, v = self._qkv(i, x)
            q, k, _ = rope(q, k, self.inv_freq, pos0=self.pos, inplace=True)
            o, _ = self.layers[i].decode(q, k, v)
            x = self._out(i, x, o)
        self.pos += 1
        return x
