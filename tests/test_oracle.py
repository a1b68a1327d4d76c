"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test pins a part of the oracle with something it does not share: a brute-force
dense formulation, a closed form, an invariant of the definition, finite differences,
torch autograd, or a torch library routine on a case that reduces to it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from tests.brute import brute_forward, torch_naive_forward
from global_attention_b200.synth import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(B, S, Hq, Hkv, D, seed=0, dout=False):
    return make_inputs(B, S, Hq=Hq, Hkv=Hkv, D=D, seed=seed, with_dout=dout)


def _problem(oracle_mod, t, **kw):
    return oracle_mod.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], **kw)


CASES = [
    # B, S, Hq, Hkv, D, R, W
    (1, 1, 4, 1, 8, 4, 3),
    (2, 37, 4, 2, 8, 4, 5),
    (1, 64, 4, 1, 128, 42, 16),
    (2, 50, 4, 1, 128, 42, 1),
    (1, 45, 8, 2, 128, 42, 45),
    (1, 30, 4, 4, 128, 0, 7),
    (1, 33, 4, 1, 128, 128, 1000),
    (1, 130, 4, 1, 128, 42, 128),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,D,R,W", CASES)
def test_forward_matches_brute_force(oracle_mod, B, S, Hq, Hkv, D, R, W):
    t = _inputs(B, S, Hq, Hkv, D, seed=S + W)
    kw = dict(rope_dims=R, rope_base=10000.0, window=W, eps=1e-6)
    out, lse = _problem(oracle_mod, t, **kw).forward()
    f = lambda x: x.to(torch.float64).numpy()
    bout, blse = brute_forward(f(t["q"]), f(t["k"]), f(t["v"]), f(t["g"]), f(t["gamma_q"]),
                               f(t["gamma_k"]), R=R, base=10000.0, W=W, eps=1e-6)
    np.testing.assert_allclose(out, bout, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, blse, rtol=0, atol=1e-12)


def test_sampled_rows_equal_full(oracle_mod):
    t = _inputs(2, 90, 8, 2, 128, seed=3, dout=True)
    P = _problem(oracle_mod, t, window=20)
    out, lse = P.forward()
    rows = np.array([0, 5, 89, 90, 131, 179])
    o2, l2 = P.forward(rows)
    b, i = rows // 90, rows % 90
    np.testing.assert_array_equal(o2, out[b, i])
    np.testing.assert_array_equal(l2, lse[b, :, i])
    full = P.backward(t["dout"])
    dq, dg = P.backward_qrows(t["dout"], rows)
    np.testing.assert_allclose(dq, full["dq"][b, i], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dg, full["dg"][b, i], rtol=0, atol=1e-13)
    dk, dv = P.backward_krows(t["dout"], rows)
    np.testing.assert_allclose(dk, full["dk"][b, i], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, full["dv"][b, i], rtol=0, atol=1e-12)


def test_window_at_least_S_is_full_causal(oracle_mod):
    """W >= S: every window is the whole causal prefix, so W = S, 2S, 10^9 agree bitwise."""
    S = 70
    t = _inputs(1, S, 4, 1, 128, seed=11)
    res = [_problem(oracle_mod, t, window=W).forward() for W in (S, 2 * S, 10**9)]
    for o, l in res[1:]:
        np.testing.assert_array_equal(o, res[0][0])
        np.testing.assert_array_equal(l, res[0][1])
    o_short, _ = _problem(oracle_mod, t, window=S - 1).forward()
    assert np.abs(o_short[0, -1] - res[0][0][0, -1]).max() > 1e-6  # last row loses key 0


def test_self_only_window(oracle_mod):
    """W = 1: out_i = sigmoid(g_i) * v_i of its own KV head; lse_i = s_ii."""
    t = _inputs(2, 20, 8, 2, 128, seed=5)
    P = _problem(oracle_mod, t, window=1)
    out, lse = P.forward()
    v = t["v"].double().numpy().repeat(4, axis=2)
    g = t["g"].double().numpy()
    np.testing.assert_allclose(out, v / (1.0 + np.exp(-g)), rtol=0, atol=1e-14)
    # lse_i = scale * q_hat_i . k_hat_i
    for (b, i, h) in [(0, 0, 0), (1, 7, 5), (1, 19, 7)]:
        qh = P.prologue_row(t["q"][b, i, h], t["gamma_q"], i)
        kh = P.prologue_row(t["k"][b, i, h // 4], t["gamma_k"], i)
        assert abs(lse[b, h, i] - np.dot(qh, kh) / math.sqrt(128)) < 1e-12


def test_zero_query_gives_window_mean(oracle_mod):
    """q = 0 -> q_hat = 0 -> uniform softmax: out_i = sigmoid(g_i) * mean of v over the
    window, lse_i = log(number of visible keys)."""
    S, W = 40, 6
    t = _inputs(1, S, 4, 2, 128, seed=6)
    t["q"] = torch.zeros_like(t["q"])
    out, lse = _problem(oracle_mod, t, window=W).forward()
    v = t["v"].double().numpy()
    g = t["g"].double().numpy()
    for i in range(S):
        lo = max(0, i - W + 1)
        mean = v[0, lo:i + 1].mean(axis=0).repeat(2, axis=0)
        np.testing.assert_allclose(out[0, i], mean / (1 + np.exp(-g[0, i])), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, :, i], math.log(i - lo + 1), rtol=0, atol=1e-14)


def test_gate_limits(oracle_mod):
    """g = +inf leaves the attention output ungated; g = 0 halves it; g = -inf zeroes it."""
    t = _inputs(1, 33, 4, 1, 128, seed=7)
    res = {}
    for name, val in (("inf", float("inf")), ("zero", 0.0), ("ninf", float("-inf"))):
        tt = dict(t)
        tt["g"] = torch.full_like(t["g"], val)
        res[name] = _problem(oracle_mod, tt, window=9).forward()[0]
    np.testing.assert_allclose(res["inf"], 2.0 * res["zero"], rtol=0, atol=1e-15)
    assert np.all(res["ninf"] == 0.0)
    f = lambda x: x.to(torch.float64).numpy()
    bout, _ = brute_forward(f(t["q"]), f(t["k"]), f(t["v"]), np.full(t["g"].shape, 60.0),
                            f(t["gamma_q"]), f(t["gamma_k"]), W=9)
    np.testing.assert_allclose(res["inf"], bout, rtol=0, atol=1e-12)


def test_rope_depends_only_on_position_difference(oracle_mod):
    t = _inputs(1, 4, 4, 1, 128, seed=8)
    P = _problem(oracle_mod, t, rope_base=10000.0)
    x, y = t["q"][0, 0, 0], t["k"][0, 1, 0]
    ref = np.dot(P.prologue_row(x, t["gamma_q"], 5), P.prologue_row(y, t["gamma_k"], 2))
    for c in (1, 17, 1000, 262000):
        d = np.dot(P.prologue_row(x, t["gamma_q"], 5 + c), P.prologue_row(y, t["gamma_k"], 2 + c))
        assert abs(d - ref) < 1e-9 * max(1.0, abs(ref))
    # the rotation is orthogonal: the norm of the normalised row is unchanged
    y0 = P.prologue_row(x, t["gamma_q"], 0)
    for pos in (1, 99, 65535):
        assert abs(np.linalg.norm(P.prologue_row(x, t["gamma_q"], pos)) - np.linalg.norm(y0)) < 1e-12
    # full causal: shifting every position by c changes nothing (rotation is relative)
    # -> out at positions 0..S-1 equals brute force with positions c..c+S-1
    # (checked through the brute-force rotation matrices, which take absolute positions)


def test_rope_pairing_closed_form(oracle_mod):
    """A one-hot row e_t (gamma = 1, eps = 0) normalises to sqrt(D) e_t; pair (t, t + R/2)
    then rotates by pos * base^(-2t/R): component t -> cos, component t+R/2 -> sin."""
    D, R, base = 128, 42, 10000.0
    t = _inputs(1, 2, 4, 1, D, seed=9)
    P = _problem(oracle_mod, t, rope_dims=R, rope_base=base, eps=0.0)
    ones = np.ones(D)
    for tt, pos in ((0, 1), (0, 3), (5, 77), (20, 1000)):
        x = np.zeros(D); x[tt] = 1.0
        y = P.prologue_row(x, ones, pos)
        a = pos * base ** (-2.0 * tt / R)
        expect = np.zeros(D)
        expect[tt] = math.sqrt(D) * math.cos(a)
        expect[tt + R // 2] = math.sqrt(D) * math.sin(a)
        np.testing.assert_allclose(y, expect, rtol=0, atol=1e-12)
    # dims at or beyond R are not rotated
    x = np.zeros(D); x[42] = 1.0; x[127] = 2.0
    y = P.prologue_row(x, ones, 12345)
    r = math.sqrt(5.0 / D)
    assert abs(y[42] - 1.0 / r) < 1e-12 and abs(y[127] - 2.0 / r) < 1e-12


def test_score_bound_of_normalised_rows(oracle_mod):
    """An RMS-normalised row has norm at most sqrt(D) before gamma (sum x^2 over mean x^2
    + eps is at most D) and the rotation keeps norms, so every score is bounded by
    |q~ . k~| <= D max|gamma_q| max|gamma_k|: the bound the sliding-window forward uses as
    its softmax reference.  Random rows of any scale stay under it; one-hot rows in an
    unrotated dimension with constant gamma and eps = 0 reach it exactly."""
    D, R = 128, 42
    t = _inputs(1, 4, 4, 1, D, seed=11)
    gq, gk = t["gamma_q"].double().numpy(), t["gamma_k"].double().numpy()
    P = _problem(oracle_mod, t, eps=1e-6)
    bound = D * np.abs(gq).max() * np.abs(gk).max()
    rng = np.random.default_rng(3)
    worst = 0.0
    for n in range(300):
        x = rng.standard_normal(D) * (1e-3, 1.0, 1e3)[n % 3]
        y = x + 0.1 * rng.standard_normal(D) if n % 2 else rng.standard_normal(D)
        a, b = rng.integers(0, 262144, 2)
        s = abs(float(np.dot(P.prologue_row(x, gq, int(a)), P.prologue_row(y, gk, int(b)))))
        assert s <= bound * (1 + 1e-12)
        worst = max(worst, s / bound)
    assert worst > 0.05  # the random rows are not trivially far from the bound
    cq, ck = 1.7, 0.6
    P0 = _problem(oracle_mod, t, eps=0.0)
    e = np.zeros(D); e[R + 5] = 3.0
    s = float(np.dot(P0.prologue_row(e, np.full(D, cq), 77), P0.prologue_row(e, np.full(D, ck), 3)))
    assert abs(s - D * cq * ck) < 1e-9 * D * cq * ck


def test_rope_base_irrelevant_when_rotated_dims_are_zero(oracle_mod):
    t = _inputs(1, 50, 4, 1, 128, seed=10)
    for name in ("q", "k"):
        x = t[name].clone(); x[..., :42] = 0; t[name] = x
    a = _problem(oracle_mod, t, rope_base=10000.0, window=13).forward()
    b = _problem(oracle_mod, t, rope_base=1.0e7, window=13).forward()
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_rmsnorm_scale_invariance(oracle_mod):
    """Scaling q (or k) by c > 0 changes only the eps term: with eps = 0 the output is
    unchanged to rounding; with eps = 1e-6 to ~1e-6 relative."""
    t = _inputs(1, 40, 4, 1, 128, seed=12)
    base = _problem(oracle_mod, t, window=11, eps=0.0).forward()[0]
    for c in (0.25, 3.0):
        tt = dict(t); tt["q"] = t["q"].double() * c; tt["k"] = t["k"].double() * (1 / c)
        o = _problem(oracle_mod, tt, window=11, eps=0.0).forward()[0]
        np.testing.assert_allclose(o, base, rtol=0, atol=1e-13)
    o_eps = _problem(oracle_mod, t, window=11, eps=1e-6).forward()[0]
    assert np.abs(o_eps - base).max() < 1e-5


def test_sdpa_special_case(oracle_mod):
    """gamma = 1, no rotation, g = +inf and eps = 0: the layer is scaled-dot-product
    attention of the RMS-normalised q, k with a banded causal mask (torch SDPA, fp64)."""
    B, S, Hq, Hkv, D, W = 2, 48, 4, 2, 128, 10
    t = _inputs(B, S, Hq, Hkv, D, seed=13)
    t["gamma_q"] = torch.ones(D); t["gamma_k"] = torch.ones(D)
    t["g"] = torch.full_like(t["g"], float("inf"))
    out, _ = _problem(oracle_mod, t, rope_dims=0, window=W, eps=0.0).forward()
    q, k, v = (t[n].double() for n in ("q", "k", "v"))
    qn = q / q.pow(2).mean(-1, keepdim=True).sqrt()
    kn = k / k.pow(2).mean(-1, keepdim=True).sqrt()
    G = Hq // Hkv
    mask = torch.ones(S, S, dtype=torch.bool).tril() & ~torch.ones(S, S, dtype=torch.bool).tril(-W)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qn.transpose(1, 2), kn.repeat_interleave(G, 2).transpose(1, 2),
        v.repeat_interleave(G, 2).transpose(1, 2), attn_mask=mask).transpose(1, 2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def _loss_grads_autograd(t, R, base, W, eps):
    scale = 1.0 / math.sqrt(t["q"].shape[-1])
    leaves = {n: t[n].double().clone().requires_grad_(True)
              for n in ("q", "k", "v", "g", "gamma_q", "gamma_k")}
    out = torch_naive_forward(leaves["q"], leaves["k"], leaves["v"], leaves["g"],
                              leaves["gamma_q"], leaves["gamma_k"], R, base, W, eps, scale)
    (out * t["dout"].double()).sum().backward()
    return {n: x.grad.numpy() for n, x in leaves.items()}


@pytest.mark.parametrize("S,W,Hq,Hkv,D,R", [(19, 4, 4, 1, 8, 4), (40, 40, 4, 2, 128, 42),
                                           (33, 7, 8, 2, 128, 42), (9, 1, 2, 1, 8, 8)])
def test_backward_matches_autograd(oracle_mod, S, W, Hq, Hkv, D, R):
    t = _inputs(2, S, Hq, Hkv, D, seed=20 + S, dout=True)
    full = _problem(oracle_mod, t, rope_dims=R, window=W, eps=1e-6).backward(t["dout"])
    ref = _loss_grads_autograd(t, R, 10000.0, W, 1e-6)
    for ours, theirs in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"),
                         ("dgamma_q", "gamma_q"), ("dgamma_k", "gamma_k")):
        np.testing.assert_allclose(full[ours], ref[theirs], rtol=1e-10, atol=1e-11, err_msg=ours)


def test_backward_finite_differences(oracle_mod):
    """Central differences of L = sum(dout * out) in fp64 on a tiny problem."""
    S, W, Hq, Hkv, D, R = 6, 3, 2, 1, 8, 4
    t = _inputs(1, S, Hq, Hkv, D, seed=31, dout=True)
    base = {n: t[n].double().numpy().copy() for n in ("q", "k", "v", "g", "gamma_q", "gamma_k")}
    dout = t["dout"].double().numpy()
    kw = dict(rope_dims=R, window=W, eps=1e-6, rope_base=100.0)

    def loss(arrs):
        o, _ = oracle_mod.Problem(arrs["q"], arrs["k"], arrs["v"], arrs["g"], arrs["gamma_q"],
                                  arrs["gamma_k"], **kw).forward()
        return float((o * dout).sum())

    full = oracle_mod.Problem(base["q"], base["k"], base["v"], base["g"], base["gamma_q"],
                              base["gamma_k"], **kw).backward(dout)
    h = 1e-6
    rng = np.random.default_rng(0)
    for ours, name in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"),
                       ("dgamma_q", "gamma_q"), ("dgamma_k", "gamma_k")):
        flat = base[name].reshape(-1)
        for idx in rng.choice(flat.size, size=min(flat.size, 12), replace=False):
            plus = {n: a.copy() for n, a in base.items()}
            minus = {n: a.copy() for n, a in base.items()}
            plus[name].reshape(-1)[idx] += h
            minus[name].reshape(-1)[idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = full[ours].reshape(-1)[idx]
            assert abs(fd - an) < 1e-7 * max(1.0, abs(an)), (ours, idx, fd, an)


def test_dgamma_dot_identity(oracle_mod):
    """gamma_q . dgamma_q = gamma_k . dgamma_k = sum_ij ds_ij s_ij (scaling q_hat by c
    and k_hat by 1/c leaves every score unchanged)."""
    t = _inputs(2, 60, 8, 2, 128, seed=40, dout=True)
    full = _problem(oracle_mod, t, window=17).backward(t["dout"])
    a = float(np.dot(full["dgamma_q"], t["gamma_q"].double().numpy()))
    b = float(np.dot(full["dgamma_k"], t["gamma_k"].double().numpy()))
    assert abs(a - b) < 1e-10 * max(1.0, abs(a))
    assert abs(a) > 1e-3


def test_dv_sum_property(oracle_mod):
    """Each query row's probabilities sum to one, so summing dv over all key rows gives
    the sum over the group's query heads and rows of dout * sigmoid(g)."""
    t = _inputs(2, 50, 8, 2, 128, seed=41, dout=True)
    full = _problem(oracle_mod, t, window=13).backward(t["dout"])
    dA = t["dout"].double().numpy() / (1 + np.exp(-t["g"].double().numpy()))
    lhs = full["dv"].sum(axis=1)                                     # [B, Hkv, D]
    rhs = dA.reshape(2, 50, 2, 4, 128).sum(axis=(1, 3))              # [B, Hkv, D]
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-11)


def test_kv_cache_golden(oracle_mod):
    """Closed-form KV-cache sizes printed on the pages (shibing624 review, section 架构)."""
    with open(os.path.join(GOLDEN, "kv_cache.json")) as f:
        gold = json.load(f)
    full = oracle_mod.kv_cache_bytes_per_token(gold["layers_total"])
    hyb = oracle_mod.kv_cache_bytes_per_token(gold["layers_global"])
    assert full == gold["full_bytes_per_token"] and hyb == gold["hybrid_bytes_per_token"]
    assert full * gold["context_tokens"] == gold["full_bytes_at_context"]
    assert hyb * gold["context_tokens"] == gold["hybrid_bytes_at_context"]
