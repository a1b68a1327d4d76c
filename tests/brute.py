"""Brute-force restatements of the layer for tiny inputs (test pins for the oracle).

These are deliberately a different formulation from the oracle: the rotation is a dense
per-position D x D matrix, the window is a dense boolean mask over all (i, j), softmax is
taken over the whole masked row with logsumexp, and GQA is an explicit head expansion.
Used only on tiny shapes (S <= a few hundred, D in {8, 128}).
"""
from __future__ import annotations

import numpy as np
import torch


def rotation_matrices(S: int, D: int, R: int, base: float) -> np.ndarray:
    """[S, D, D]: rot[pos] @ y rotates pairs (t, t+R/2) by pos * base^(-2t/R)."""
    rot = np.tile(np.eye(D), (S, 1, 1))
    half = R // 2
    for t in range(half):
        theta = base ** (-2.0 * t / R)
        for pos in range(S):
            a = pos * theta
            c, s = np.cos(a), np.sin(a)
            rot[pos, t, t] = c
            rot[pos, t, t + half] = -s
            rot[pos, t + half, t] = s
            rot[pos, t + half, t + half] = c
    return rot


def window_mask(S: int, W: int) -> np.ndarray:
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    return (j <= i) & (j > i - W)


def brute_forward(q, k, v, g, gamma_q, gamma_k, R=42, base=10000.0, W=128, eps=1e-6, scale=None):
    """Dense numpy forward: returns out [B,S,Hq,D], lse [B,Hq,S]."""
    q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g))
    gamma_q = np.asarray(gamma_q, dtype=np.float64)
    gamma_k = np.asarray(gamma_k, dtype=np.float64)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)

    def norm(x, gamma):
        return gamma * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)

    rot = rotation_matrices(S, D, R, base)
    qh = np.einsum("sde,bshe->bshd", rot, norm(q, gamma_q))
    kh = np.einsum("sde,bshe->bshd", rot, norm(k, gamma_k))
    kh = np.repeat(kh, G, axis=2)            # head h reads KV head h // G
    ve = np.repeat(v, G, axis=2)
    scores = scale * np.einsum("bihd,bjhd->bhij", qh, kh)
    mask = window_mask(S, W)
    scores = np.where(mask[None, None], scores, -np.inf)
    m = scores.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.exp(scores - m).sum(axis=-1, keepdims=True)))[..., 0]
    P = np.exp(scores - lse[..., None])
    A = np.einsum("bhij,bjhd->bihd", P, ve)
    out = A / (1.0 + np.exp(-g))
    return out, lse


def torch_naive_forward(q, k, v, g, gamma_q, gamma_k, R, base, W, eps, scale):
    """The same layer in fp64 torch ops (autograd-able), for gradient pins."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    rot = torch.from_numpy(rotation_matrices(S, D, R, base))

    def norm(x, gamma):
        return gamma * x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + eps)

    qh = torch.einsum("sde,bshe->bshd", rot, norm(q, gamma_q))
    kh = torch.einsum("sde,bshe->bshd", rot, norm(k, gamma_k)).repeat_interleave(G, dim=2)
    ve = v.repeat_interleave(G, dim=2)
    s = scale * torch.einsum("bihd,bjhd->bhij", qh, kh)
    mask = torch.from_numpy(window_mask(S, W))
    s = s.masked_fill(~mask, float("-inf"))
    p = torch.softmax(s, dim=-1)
    A = torch.einsum("bhij,bjhd->bihd", p, ve)
    return torch.sigmoid(g) * A
