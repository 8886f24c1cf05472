"""A Gated DeltaNet-2 layer around the operator: input projection, gate activations, the Gated Delta Rule-2,
output projection.

The pages name the layer's parts only as the operator plus "two additional per-channel gate computations"
(GitHub README method bullets; aiexpert.news article) next to KDA's channel-wise decay. This module takes the
plainest reading (the same as the library's gate kernels, ``gdn2_layer_gates_fwd``):

    z = x W_in  ->  q, k (L2-normalised per head), v, b = sigmoid, w = sigmoid, log_alpha = -softplus(z_a + a_bias)
    o, S_T = Gated Delta Rule-2 (q, k, v, log_alpha, b, w, S0)
    y = o W_out

The projections are plain GEMMs (cuBLAS through torch.matmul); the gate activations, the operator and their
backward run in the library's kernels. Short convolutions, output normalisation and gating, and the hybrid
sliding-window layers of the pages' models are not part of this reading.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import binding


class LayerGates(torch.autograd.Function):
    """Gate activations through the library's kernels (forward and backward)."""

    @staticmethod
    def forward(ctx, z, a_bias, Dk, Dv):
        z = z.contiguous()
        out = binding.gdn2_layer_gates_fwd(z, Dk, Dv, a_bias)
        ctx.save_for_backward(z, a_bias if a_bias is not None else torch.empty(0))
        ctx.has_bias, ctx.Dk, ctx.Dv = a_bias is not None, Dk, Dv
        return out

    @staticmethod
    def backward(ctx, dq, dk, dv, db, dw, dla):
        z, a_bias = ctx.saved_tensors
        a_bias = a_bias if ctx.has_bias else None
        grads = [g.contiguous() if g is not None else torch.zeros(z.shape[:3] + (D,), dtype=z.dtype, device=z.device)
                 for g, D in zip((dq, dk, dv, db, dw, dla), (ctx.Dk, ctx.Dk, ctx.Dv, ctx.Dk, ctx.Dv, ctx.Dk))]
        dz = binding.gdn2_layer_gates_bwd(z, *grads, ctx.Dk, ctx.Dv, a_bias)
        da = None
        if ctx.has_bias:   # the bias gradient: dz_a summed over batch and tokens
            da = dz[..., 3 * ctx.Dk + 2 * ctx.Dv:].float().sum((0, 1))
        return dz, da, None, None


class Gdn2Layer(torch.nn.Module):
    """``y, S_T = layer(x, S0)`` for x [B, T, d_model]; bf16 (tensor-core operator path at d = 128) or fp32."""

    def __init__(self, d_model: int, n_heads: int, d_k: int = 128, d_v: int = 128, chunk: int = 64,
                 dtype=torch.bfloat16, device=None, decay_bias: float = -4.0):
        super().__init__()
        self.d_model, self.H, self.Dk, self.Dv, self.chunk = d_model, n_heads, d_k, d_v, chunk
        width = n_heads * (4 * d_k + 2 * d_v)
        self.W_in = torch.nn.Parameter(torch.randn(d_model, width, device=device).div_(math.sqrt(d_model)).to(dtype))
        self.W_out = torch.nn.Parameter(torch.randn(n_heads * d_v, d_model, device=device)
                                        .div_(math.sqrt(n_heads * d_v)).to(dtype))
        # softplus(-4) ~ 0.018: a slow resting decay per token
        self.a_bias = torch.nn.Parameter(torch.full((n_heads, d_k), float(decay_bias), device=device))

    def forward(self, x, S0: Optional[torch.Tensor] = None):
        B, T, _ = x.shape
        z = (x @ self.W_in).view(B, T, self.H, 4 * self.Dk + 2 * self.Dv)
        q, k, v, b, w, la = LayerGates.apply(z, self.a_bias, self.Dk, self.Dv)
        o, ST = binding.gated_delta_rule2(q, k, v, la, b, w, S0, self.chunk)
        y = o.reshape(B, T, self.H * self.Dv) @ self.W_out
        return y, ST
