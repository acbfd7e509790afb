"""RACE attention as a differentiable multi-head attention layer.

The pages scale-test RACE as the attention of a multi-head layer trained end to end
([ABS]: a forward-backward pass of a multi-head attention layer; [JA] §2.2: the soft
assignment with its temperature is differentiable, so the sketch trains with the rest
of the model).  This module wraps the C ABI for that use:

* ``RaceAttentionFunction`` — a ``torch.autograd.Function`` whose forward calls
  ``race_forward_ex`` (saving den) and whose backward calls ``race_backward_ex``; it
  returns gradients for q, k, v and the hash planes W.
* ``RaceMultiHeadAttention`` — q/k/v/o projections (plain GEMMs, as in any attention
  layer) around RACE attention over ``heads`` heads of size 64.  The hash planes W are a
  parameter (trained with the rest when ``learn_planes``) or a fixed buffer, either shared
  by all heads ([L, 64, P]) or one set per head ([heads, L, 64, P]).

Every RACE step runs in the library's kernels; this module only reshapes and marshals.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import race_attn as ra


class RaceAttentionFunction(torch.autograd.Function):
    """out = RACE(q, k, v; W) for q, k, v of shape [H, N, 64] (contiguous) and W of shape
    [L, 64, P] (shared) or [H, L, 64, P] (per head), float32."""

    @staticmethod
    def forward(ctx, q, k, v, W, tau: float, causal: bool, impl: str = "auto"):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        W = W.contiguous()
        out, den = ra.forward(q, k, v, W, tau, causal, return_den=True, impl=impl)
        ctx.save_for_backward(q, k, v, W, out, den)
        ctx.tau, ctx.causal, ctx.impl = tau, causal, impl
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, W, out, den = ctx.saved_tensors
        dq, dk, dv, dW = ra.backward(q, k, v, W, ctx.tau, ctx.causal, out,
                                     dout.contiguous().to(q.dtype), den=den, impl=ctx.impl)
        return dq, dk, dv, dW, None, None, None


def race_attention(q, k, v, W, tau: float, causal: bool, impl: str = "auto"):
    """Functional form of RaceAttentionFunction."""
    return RaceAttentionFunction.apply(q, k, v, W, tau, causal, impl)


class RaceMultiHeadAttention(torch.nn.Module):
    """Multi-head attention layer with RACE attention over heads of size 64.

    x: [B, N, d_model] -> y: [B, N, d_model].  q, k, v = x Wq, x Wk, x Wv split into
    ``heads`` heads; each (batch, head) pair is one head of the library; y = o Wo.
    """

    head_dim = 64

    def __init__(self, d_model: int, heads: int, L: int, P: int, tau: float,
                 causal: bool = True, learn_planes: bool = True, per_head_planes: bool = False,
                 bias: bool = False, impl: str = "auto", device=None, dtype=torch.bfloat16,
                 seed: Optional[int] = None):
        super().__init__()
        self.d_model, self.heads, self.L, self.P = d_model, heads, L, P
        self.tau, self.causal, self.impl = float(tau), bool(causal), impl
        self.per_head_planes = per_head_planes
        inner = heads * self.head_dim
        kw = dict(device=device, dtype=dtype)
        self.wq = torch.nn.Linear(d_model, inner, bias=bias, **kw)
        self.wk = torch.nn.Linear(d_model, inner, bias=bias, **kw)
        self.wv = torch.nn.Linear(d_model, inner, bias=bias, **kw)
        self.wo = torch.nn.Linear(inner, d_model, bias=bias, **kw)
        gen = torch.Generator(device="cpu")
        if seed is not None:
            gen.manual_seed(seed)
        shape = (heads, L, self.head_dim, P) if per_head_planes else (L, self.head_dim, P)
        planes = torch.randn(shape, generator=gen, dtype=torch.float32).to(device)
        if learn_planes:
            self.planes = torch.nn.Parameter(planes)
        else:
            self.register_buffer("planes", planes)

    def _split(self, t, B, N):
        # [B, N, heads * 64] -> [B * heads, N, 64]
        return t.view(B, N, self.heads, self.head_dim).transpose(1, 2).reshape(
            B * self.heads, N, self.head_dim)

    def _planes_for(self, B):
        if not self.per_head_planes:
            return self.planes
        # one set of planes per head, repeated over the batch: [B * heads, L, 64, P]
        return self.planes.unsqueeze(0).expand(B, *self.planes.shape).reshape(
            B * self.heads, self.L, self.head_dim, self.P)

    def forward(self, x):
        B, N, _ = x.shape
        q = self._split(self.wq(x), B, N)
        k = self._split(self.wk(x), B, N)
        v = self._split(self.wv(x), B, N)
        o = race_attention(q, k, v, self._planes_for(B), self.tau, self.causal, self.impl)
        o = o.view(B, self.heads, N, self.head_dim).transpose(1, 2).reshape(
            B, N, self.heads * self.head_dim)
        return self.wo(o)

    def extra_repr(self) -> str:
        return (f"d_model={self.d_model}, heads={self.heads}, L={self.L}, P={self.P}, "
                f"tau={self.tau}, causal={self.causal}, per_head_planes={self.per_head_planes}")


def init_like_attention(layer: RaceMultiHeadAttention):
    """Scaled-normal projection weights (std 1/sqrt(fan_in)), as is usual for attention."""
    with torch.no_grad():
        for lin in (layer.wq, layer.wk, layer.wv, layer.wo):
            lin.weight.normal_(0.0, 1.0 / math.sqrt(lin.in_features))
            if lin.bias is not None:
                lin.bias.zero_()
    return layer
