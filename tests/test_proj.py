"""Projections around the attention layer on the B200 against the fp64 oracle (oracle/proj.py),
through the C ABI (include/zgcm_proj.h).

Tolerance, from the arithmetic: each output element is one bf16 rounding (relative 2^-9) of an
fp32 sum of exact bf16 products, so against the fp64 product of the same bf16 inputs it is
within 2^-8 |ref| plus the fp32 summation error, bounded with margin by 2^-18 times the sum of
the products' magnitudes.
"""
import numpy as np
import pytest
import torch

import global_attention_b200 as ga
from oracle import proj

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ga.load()


def _r(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _close(name, got, ref, mag):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref) - (2.0 ** -8 * np.abs(ref) + 2.0 ** -18 * mag)
    assert np.all(err <= 0), (name, float(err.max()))


# (T tokens, d_model, Hq, Hkv, D): a ragged token count, the model's head layout at a smaller
# hidden size, and T not a multiple of 8 (the weight gradients sum over the tokens)
CASES = [(300, 512, 4, 2, 128), (1000, 1024, 8, 2, 128), (77, 256, 2, 2, 128)]


@pytest.mark.parametrize("T,dm,Hq,Hkv,D", CASES)
def test_qkvg_projection(T, dm, Hq, Hkv, D):
    wq, wkv = Hq * D, Hkv * D
    x = _r((T, dm), T)
    w = _r((2 * (wq + wkv), dm), dm, dm ** -0.5)
    parts = ga.zgcm_proj_qkvg_fwd(x.cuda(), w.cuda(), Hq=Hq, Hkv=Hkv, D=D)
    torch.cuda.synchronize()
    ref = proj.qkvg_forward(x, w, wq, wkv)
    xa, wa = np.abs(x.double().numpy()), np.abs(w.double().numpy())
    mags = np.split(xa @ wa.T, [wq, wq + wkv, wq + 2 * wkv], axis=1)
    for n, got, r, m in zip(("q", "k", "v", "g"), parts, ref, mags):
        assert got.shape == r.shape, n
        _close(n, got, r, m)
    grads = [_r(p.shape, 50 + i) for i, p in enumerate(parts)]
    dx, dw = ga.zgcm_proj_qkvg_bwd(x.cuda(), w.cuda(), *(g.cuda() for g in grads), Hq=Hq, Hkv=Hkv, D=D)
    torch.cuda.synchronize()
    rdx, rdw = proj.qkvg_backward(x, w, *grads)
    ga_ = np.abs(np.concatenate([g.double().numpy() for g in grads], axis=1))
    _close("dx", dx, rdx, ga_ @ wa)
    _close("dw", dw, rdw, ga_.T @ xa)


@pytest.mark.parametrize("T,din,dm", [(300, 512, 768), (77, 256, 256), (1000, 1024, 1024)])
def test_output_projection(T, din, dm):
    a = _r((T, din), T + 1)
    w = _r((dm, din), din, din ** -0.5)
    y = ga.zgcm_proj_out_fwd(a.cuda(), w.cuda())
    dy = _r((T, dm), 9)
    da, dw = ga.zgcm_proj_out_bwd(a.cuda(), w.cuda(), dy.cuda())
    torch.cuda.synchronize()
    aa, wa, dya = (np.abs(t.double().numpy()) for t in (a, w, dy))
    _close("y", y, proj.out_forward(a, w), aa @ wa.T)
    rda, rdw = proj.out_backward(a, w, dy)
    _close("da", da, rda, dya @ wa)
    _close("dw", dw, rdw, dya.T @ aa)
