"""Seeded synthetic inputs for the gated window-attention layer.

This module holds no arithmetic of the layer: it only draws random tensors and picks
sample rows.  It is the one piece the GPU path and the fp64 oracle share.

Recipe: a CPU ``torch.Generator`` seeded with ``seed + offset`` per tensor
(q +0, k +1, v +2, g +3, gamma_q +4, gamma_k +5, dout +6); q, k, v, g and dout are
standard normal drawn in fp32 and rounded to bf16 (round-to-nearest-even); gamma_q and
gamma_k are uniform on [0.5, 1.5) in fp32.
"""
from __future__ import annotations

import numpy as np
import torch

OFFSETS = dict(q=0, k=1, v=2, g=3, gamma_q=4, gamma_k=5, dout=6)


def _gen(seed: int, name: str) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed) + OFFSETS[name])


def make_inputs(B: int, S: int, Hq: int = 32, Hkv: int = 8, D: int = 128, seed: int = 0,
                with_dout: bool = False) -> dict:
    """CPU tensors: q, g [B,S,Hq,D] bf16; k, v [B,S,Hkv,D] bf16; gamma_q, gamma_k [D] fp32;
    dout [B,S,Hq,D] bf16 when with_dout."""
    t = {}
    for name, shape in (("q", (B, S, Hq, D)), ("k", (B, S, Hkv, D)), ("v", (B, S, Hkv, D)),
                        ("g", (B, S, Hq, D))):
        t[name] = torch.randn(shape, generator=_gen(seed, name), dtype=torch.float32).to(torch.bfloat16)
    for name in ("gamma_q", "gamma_k"):
        t[name] = torch.rand((D,), generator=_gen(seed, name), dtype=torch.float32) + 0.5
    if with_dout:
        t["dout"] = torch.randn((B, S, Hq, D), generator=_gen(seed, "dout"),
                                dtype=torch.float32).to(torch.bfloat16)
    return t


def sample_query_rows(B: int, S: int, n_random: int, edge: int = 256, block: int = 128,
                      seed: int = 0) -> np.ndarray:
    """Flat row indices b*S+i to check at full size: the first and last `edge` positions of
    the first and last sequence, positions on either side of every `block` boundary that
    falls in that range, and `n_random` seeded positions anywhere."""
    rng = np.random.default_rng(seed + 1000)
    rows = set()
    for b in {0, B - 1}:
        for i in list(range(min(edge, S))) + list(range(max(0, S - edge), S)):
            rows.add(b * S + i)
    for _ in range(n_random):
        rows.add(int(rng.integers(0, B)) * S + int(rng.integers(0, S)))
    for b in {0, B - 1}:
        for c in range(block, S, block * max(1, S // (block * 16))):
            for i in (c - 1, c):
                rows.add(b * S + i)
    return np.array(sorted(r for r in rows if 0 <= r < B * S), dtype=np.int64)
