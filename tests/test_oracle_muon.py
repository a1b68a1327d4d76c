"""Pins of the Muon oracle (oracle/muon.py) against what the mathematics fixes, so that a
plausible slip in it (a dropped term, a wrong power or coefficient, a missing transpose, the
norm or the update formula) fails here before any GPU result is compared with it."""
import numpy as np
import pytest

from oracle import muon


def _svd_matrix(m, n, s, seed):
    """U diag(s) V^T with random orthonormal U (m x r), V (n x r), r = len(s)."""
    rng = np.random.default_rng(seed)
    r = len(s)
    U, _ = np.linalg.qr(rng.standard_normal((m, r)))
    V, _ = np.linalg.qr(rng.standard_normal((n, r)))
    return U, V, U @ np.diag(s) @ V.T


@pytest.mark.parametrize("m,n,coeffs", [(6, 9, (1.5, -0.5, 0.0)), (9, 6, (1.5, -0.5, 0.0)),
                                        (5, 5, (2.0, -1.5, 0.5)), (4, 11, (3.0, -3.2, 1.2))])
def test_singular_values_follow_the_polynomial(m, n, coeffs):
    """Every step maps X = U S V^T to U p(S) V^T with p(s) = a s + b s^3 + c s^5 (X X^T = U S^2
    U^T commutes through), so after k steps the singular vectors are unchanged and each
    singular value is p applied k times to s / ||s||_2 (||G||_F = ||s||_2).  Computed here
    on the scalars alone."""
    a, b, c = coeffs
    r = min(m, n)
    s = np.linspace(1.0, 0.1, r)
    U, V, G = _svd_matrix(m, n, s, seed=m * 31 + n)
    x = s / np.linalg.norm(s)
    for _ in range(5):
        x = a * x + b * x ** 3 + c * x ** 5
    want = U @ np.diag(x) @ V.T
    got = muon.newton_schulz(G, 5, coeffs, eps=0.0)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_transpose_symmetry():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((7, 12))
    assert np.allclose(muon.newton_schulz(G.T), muon.newton_schulz(G).T, rtol=0, atol=1e-14)


def test_many_steps_reach_the_polar_factor():
    """With the classical coefficients the iteration converges to the orthogonal polar factor
    U V^T (every singular value to 1) from any start with singular values in (0, sqrt 3)."""
    rng = np.random.default_rng(5)
    G = rng.standard_normal((8, 13))
    U, _, Vt = np.linalg.svd(G, full_matrices=False)
    got = muon.newton_schulz(G, 60)
    assert np.allclose(got, U @ Vt, rtol=0, atol=1e-10)
    assert np.allclose(got @ got.T, np.eye(8), rtol=0, atol=1e-10)


def test_zero_steps_is_the_normalised_input():
    G = np.arange(1.0, 7.0).reshape(2, 3)
    assert np.allclose(muon.newton_schulz(G, 0, eps=0.0), G / np.sqrt(91.0), rtol=0, atol=1e-15)


def test_step_update_by_hand():
    """M' = 0.9 M + G; W' = W (1 - lr wd) - lr O, O = NS(M') (here zero steps: M' / ||M'||_F)."""
    W = np.array([[1.0, -2.0], [0.5, 4.0]])
    G = np.array([[3.0, 0.0], [0.0, 4.0]])
    M = np.array([[10.0, 0.0], [0.0, 0.0]])
    W2, M2 = muon.muon_step(W, G, M, lr=0.5, weight_decay=0.2, momentum=0.9, steps=0, eps=0.0)
    assert np.allclose(M2, [[12.0, 0.0], [0.0, 4.0]])
    O = np.array([[12.0, 0.0], [0.0, 4.0]]) / np.sqrt(160.0)
    assert np.allclose(W2, W * 0.9 - 0.5 * O, rtol=0, atol=1e-15)


def test_pages_constants():
    """ZGCM-1 summary, section "前置知识 / Muon 优化器": momentum 0.9, five iterations, learning
    rate 2e-4, weight decay 0.1."""
    assert (muon.MOMENTUM, muon.NS_STEPS, muon.LR, muon.WEIGHT_DECAY) == (0.9, 5, 2e-4, 0.1)


def test_flop_count():
    # 5 steps of X X^T (2 p^2 q) and (.) X (2 p^2 q), plus A A (2 p^3) for a quintic
    assert muon.ns_flops(4, 10) == 5 * 4 * 16 * 10
    assert muon.ns_flops(10, 4, quintic=True) == 5 * (4 * 16 * 10 + 2 * 64)
