"""A causal self-attention block whose attention is the Lighthouse layer.

x [B, N, d_model] -> fused Q/K/V projection -> H heads of width d -> Lighthouse
attention (pyramid, scores, joint top-S, dense causal attention on the selected
sub-sequence, scatter-back; the C-ABI library's lh_forward / lh_backward) ->
output projection.  The pages put Lighthouse Attention in place of the
attention of a Llama-3-style decoder and train it at 98,304 tokens of context
(gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto Largo mediante
Atención Lighthouse", §2 and §4); the projections here are plain cuBLAS GEMMs
(torch.nn.Linear), the attention is the library's kernels.  No positional
encoding is applied: the layer scores and attends the projections it is given.
"""
from __future__ import annotations

import torch

from . import lighthouse as lh


class LighthouseBlock(torch.nn.Module):
    def __init__(self, d_model: int, n_heads: int, p: int, L: int, S: int, scale: float = 0.0,
                 options=None, device=None, dtype=torch.bfloat16):
        super().__init__()
        if d_model % n_heads:
            raise ValueError("d_model must be a multiple of n_heads")
        self.d_model, self.n_heads, self.head_dim = d_model, n_heads, d_model // n_heads
        self.p, self.L, self.S, self.scale, self.options = p, L, S, scale, options
        self.wqkv = torch.nn.Linear(d_model, 3 * d_model, bias=False, device=device, dtype=dtype)
        self.wo = torch.nn.Linear(d_model, d_model, bias=False, device=device, dtype=dtype)

    def split_heads(self, x):
        """q, k, v [B, H, N, d] (contiguous) from x [B, N, d_model]."""
        B, N, _ = x.shape
        qkv = self.wqkv(x).view(B, N, 3, self.n_heads, self.head_dim).permute(2, 0, 3, 1, 4)
        return qkv[0].contiguous(), qkv[1].contiguous(), qkv[2].contiguous()

    def forward(self, x):
        B, N, _ = x.shape
        q, k, v = self.split_heads(x)
        o = lh.LighthouseAttention.apply(q, k, v, self.p, self.L, self.S, self.scale, self.options)
        return self.wo(o.transpose(1, 2).reshape(B, N, self.d_model))


class DenseBlock(LighthouseBlock):
    """The same block with dense causal attention (torch SDPA), for comparison."""

    def forward(self, x):
        B, N, _ = x.shape
        q, k, v = self.split_heads(x)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
        return self.wo(o.transpose(1, 2).reshape(B, N, self.d_model))
