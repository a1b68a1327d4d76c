"""Muon optimiser step on the B200 against the fp64 oracle (oracle/muon.py), through the C ABI
(include/zgcm_muon.h).

Tolerances, from the arithmetic: the product kernel rounds its output once to bf16 (relative
2^-9) from fp32 sums of exact bf16 products, so against the fp64 product of the same bf16
inputs every element is within 2^-8 |C| + a small multiple of the fp32 summation error.  The
iteration rounds each of its three products per step to bf16 and starts from a bf16 X0; the
errors stay of the size of one bf16 rounding per product, unamplified, because every step maps
singular values below 1 to values below 1 (the polynomial is a contraction near its fixed
point): over 5 steps a relative Frobenius error within 2e-2 of the exact iterate.
"""
import numpy as np
import pytest
import torch

import global_attention_b200 as ga
from oracle import muon

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ga.load()


def _randn(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _rel_fro(got, ref):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


# (M, N, K, B given as [K, N]): single tiles, ragged tiles in every direction, K not a
# multiple of the 64-wide stage, both operand layouts
GEMM_CASES = [(128, 256, 64, False), (128, 256, 64, True), (200, 264, 136, False), (200, 264, 136, True),
              (384, 520, 1000, True), (72, 8, 8, False), (513, 1032, 2048, False)]


@pytest.mark.parametrize("M,N,K,kn", GEMM_CASES)
def test_gemm_matches_fp64_product(M, N, K, kn):
    A = _randn((M, K), 1 + M)
    B = _randn((K, N) if kn else (N, K), 2 + N)
    D = _randn((M, N), 3 + K)
    alpha, beta = 0.75, -1.25
    C = ga.zgcm_muon_gemm(A.cuda(), B.cuda(), D=D.cuda(), alpha=alpha, beta=beta, b_kn=kn)
    torch.cuda.synchronize()
    a, b, d = (x.double().numpy() for x in (A, B, D))
    ref = alpha * (a @ (b if kn else b.T)) + beta * d
    got = C.double().cpu().numpy()
    # one bf16 rounding of the result, plus the fp32 summation of K exact products (bounded by
    # a few units of 2^-24 times the sum of their magnitudes, with margin)
    mag = np.abs(alpha) * (np.abs(a) @ np.abs(b if kn else b.T)) + np.abs(beta * d)
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -18 * mag
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


# (m, n, coefficients): wide, tall (transposed path), square, a quintic with every term, and the
# largest shapes of the model's matrices at reduced width
NS_CASES = [(256, 512, (1.5, -0.5, 0.0)), (512, 200, (1.5, -0.5, 0.0)), (1024, 1024, (1.5, -0.5, 0.0)),
            (384, 640, (2.0, -1.5, 0.5)), (1024, 2752, (1.5, -0.5, 0.0))]


@pytest.mark.parametrize("m,n,coeffs", NS_CASES)
def test_orthogonalize_matches_oracle(m, n, coeffs):
    G = _randn((m, n), 7 + m + n)
    out = ga.zgcm_muon_orthogonalize(G.cuda(), steps=5, coeffs=coeffs)
    torch.cuda.synchronize()
    assert ga.zgcm_attn_device_error() == 0
    ref = muon.newton_schulz(G, 5, coeffs, eps=1e-7)
    err = _rel_fro(out, ref)
    assert err <= 2e-2, err


def test_orthogonalize_follows_the_singular_values():
    """Singular values of the GPU iterate against the closed form p^5(s / ||s||)."""
    m, n = 256, 384
    rng = np.random.default_rng(11)
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, m)))
    s = np.linspace(2.0, 0.5, m)
    G = torch.from_numpy(U @ np.diag(s) @ V.T).to(torch.bfloat16)
    out = ga.zgcm_muon_orthogonalize(G.cuda(), steps=5).double().cpu().numpy()
    x = np.linalg.svd(G.double().numpy(), compute_uv=False)
    x = x / np.linalg.norm(x)
    for _ in range(5):
        x = 1.5 * x - 0.5 * x ** 3
    got = np.linalg.svd(out, compute_uv=False)
    assert np.max(np.abs(got - x) / x) < 2e-2


@pytest.mark.parametrize("m,n", [(256, 512), (640, 384)])
def test_step_matches_oracle(m, n):
    """The whole step: momentum buffer to fp32 rounding, W to the update's error times lr."""
    W = torch.randn((m, n), generator=torch.Generator().manual_seed(m)) * 0.02
    G = _randn((m, n), 100 + n, 0.01)
    M = torch.randn((m, n), generator=torch.Generator().manual_seed(n)) * 0.005
    lr, wd = 2e-2, 0.1  # a larger lr than the pages' 2e-4, so the update dominates W's rounding
    W2, M2 = ga.zgcm_muon_step(W.cuda(), G.cuda(), M.cuda(), lr=lr, weight_decay=wd, momentum=0.9)
    torch.cuda.synchronize()
    refW, refM = muon.muon_step(W, G, M, lr=lr, weight_decay=wd, momentum=0.9)
    assert np.allclose(M2.double().cpu().numpy(), refM, rtol=1e-6, atol=1e-9)
    O_ref = muon.newton_schulz(refM, 5)
    O_got = (W.double().numpy() * (1 - lr * wd) - W2.double().cpu().numpy()) / lr
    assert _rel_fro(O_got, O_ref) <= 2e-2


def test_step_is_deterministic():
    m, n = 512, 768
    G = _randn((m, n), 5).cuda()
    res = []
    for _ in range(2):
        W = torch.ones((m, n), device="cuda") * 0.01
        M = torch.zeros((m, n), device="cuda")
        ga.zgcm_muon_step(W, G, M)
        res.append(W.clone())
    torch.cuda.synchronize()
    assert torch.equal(res[0], res[1])
