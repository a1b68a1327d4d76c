"""fp64 CPU oracle of the Muon optimiser step for one matrix parameter (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this module; it shares no code with the GPU library.  Plain numpy in float64, the steps in the
order the pages give them, one library matmul per product.

What the pages fix (ZGCM-1 summary, section "前置知识 / Muon 优化器"; shibing624 review,
section "⚙️ 训练系统"): matrix parameters take Muon with momentum 0.9, a spectral-norm
scaling, five Newton–Schulz iterations, learning rate 2e-4 and weight decay 0.1 (scalar
parameters stay on Adam, outside this module).  Readings where they are silent:

* momentum: the plain accumulation M <- mu M + G, and the step orthogonalises M;
* spectral-norm scaling: the iteration starts from X0 = M / (||M||_F + eps) — the Frobenius
  norm bounds the spectral norm, so every singular value of X0 is at most 1;
* Newton–Schulz iteration: the odd polynomial X <- a X + b (X X^T) X + c (X X^T)^2 X, written
  with A = X X^T as X <- a X + (b A + c A A) X, on the wide orientation (a tall matrix is
  transposed first and the result transposed back).  The pages give no coefficients; the
  default is the classical Newton–Schulz step for the orthogonal polar factor,
  (a, b, c) = (1.5, -0.5, 0), and any (a, b, c) may be passed;
* update: decoupled weight decay, W <- W (1 - lr wd) - lr O, O the orthogonalised momentum;
  no further scale on O (the pages name none).

Pinned by ``tests/test_oracle_muon.py`` (closed form through the singular value decomposition,
transpose symmetry, convergence to the polar factor, a hand-computed update).
"""
from __future__ import annotations

import numpy as np

# ZGCM-1 summary, "前置知识 / Muon 优化器": momentum 0.9, five Newton–Schulz steps, lr 2e-4,
# weight decay 0.1
MOMENTUM = 0.9
NS_STEPS = 5
LR = 2e-4
WEIGHT_DECAY = 0.1
# the classical Newton–Schulz step X <- 1.5 X - 0.5 X X^T X (a reading: the pages give none)
NS_COEFFS = (1.5, -0.5, 0.0)
EPS = 1e-7


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to(torch.float64).cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def newton_schulz(G, steps: int = NS_STEPS, coeffs=NS_COEFFS, eps: float = EPS) -> np.ndarray:
    """Orthogonalise G (m x n): X0 = G / (||G||_F + eps), then `steps` iterations of
    X <- a X + (b A + c A A) X with A = X X^T on the orientation with fewer rows."""
    a, b, c = coeffs
    X = _f64(G)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    X = X / (np.sqrt(np.sum(X * X)) + eps)
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if tall else X


def muon_step(W, G, M, *, lr: float = LR, weight_decay: float = WEIGHT_DECAY, momentum: float = MOMENTUM,
              steps: int = NS_STEPS, coeffs=NS_COEFFS, eps: float = EPS):
    """One Muon step of one matrix parameter: returns (W', M') from W, its gradient G and the
    momentum buffer M (all m x n)."""
    M_new = momentum * _f64(M) + _f64(G)
    O = newton_schulz(M_new, steps, coeffs, eps)
    W_new = _f64(W) * (1.0 - lr * weight_decay) - lr * O
    return W_new, M_new


def ns_flops(m: int, n: int, steps: int = NS_STEPS, quintic: bool = False) -> int:
    """Multiply-add FLOPs (2 per multiply-add) of the iterations on an m x n matrix (p = min,
    q = max): X X^T is 2 p^2 q, A A is 2 p^3 (when c != 0), (.) X is 2 p^2 q per step."""
    p, q = min(m, n), max(m, n)
    return steps * (4 * p * p * q + (2 * p ** 3 if quintic else 0))
