"""PyTorch autograd entry point of the layer: out = zgcm_attention(q, k, v, g, gamma_q,
gamma_k, window=...) in a training graph, backward included.

The forward runs the training pair that keeps activations where it applies (the normalised,
rotated q~, k~ and every row's inverse RMS stay in a store that the backward reads instead of
converting q and k again; bit-identical to the plain pair), and the plain pair elsewhere.
Argument marshalling only: both passes are the library's kernels.  Gradients flow to q, k,
v, g, gamma_q and gamma_k; lse is kept for the backward and not returned.

`ops` (tests only) replaces the three calls (forward, backward, store size) with others of the
same signatures, so that the plumbing can be checked on the CPU.
"""
from __future__ import annotations

import math

import torch


def _default_ops():
    import global_attention_b200 as ga
    return ga.zgcm_attn_fwd, ga.zgcm_attn_bwd, ga.zgcm_attn_saved_size


class ZgcmAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, gamma_q, gamma_k, window, rope_dims, rope_base, eps, scale, ops):
        fwd, bwd, saved_size = ops
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        kw = dict(rope_dims=rope_dims, rope_base=rope_base, window=window, eps=eps, scale=scale)
        n = saved_size(B, S, Hq, Hkv, D, rope_dims, window)
        store = torch.empty(n, dtype=torch.uint8, device=q.device) if n > 0 else None
        if store is not None:
            out, lse = fwd(q, k, v, g, gamma_q, gamma_k, saved=store, **kw)
        else:
            out, lse = fwd(q, k, v, g, gamma_q, gamma_k, **kw)
        ctx.save_for_backward(q, k, v, g, gamma_q, gamma_k, out, lse,
                              store if store is not None else torch.empty(0, dtype=torch.uint8))
        ctx.has_store, ctx.kw, ctx.bwd = store is not None, kw, bwd
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        q, k, v, g, gamma_q, gamma_k, out, lse, store = ctx.saved_tensors
        extra = dict(saved=store) if ctx.has_store else {}
        gr = ctx.bwd(q, k, v, g, gamma_q, gamma_k, out, lse, dout.contiguous(), **ctx.kw, **extra)
        return (gr["dq"], gr["dk"], gr["dv"], gr["dg"], gr["dgamma_q"], gr["dgamma_k"],
                None, None, None, None, None, None)


def zgcm_attention(q, k, v, g, gamma_q, gamma_k, *, window=128, rope_dims=42, rope_base=10000.0, eps=1e-6,
                   scale=None, return_lse=False, ops=None):
    """Gated window attention with autograd: q, g [B,S,Hq,D], k, v [B,S,Hkv,D] (bf16, CUDA),
    gamma_q, gamma_k [D] fp32.  Returns out [B,S,Hq,D] (and lse [B,Hq,S] with return_lse)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    out, lse = ZgcmAttentionFunction.apply(q, k, v, g, gamma_q, gamma_k, int(window), int(rope_dims),
                                           float(rope_base), float(eps), float(scale), ops or _default_ops())
    return (out, lse) if return_lse else out
