"""global_attention_b200.autograd: the plumbing of the autograd entry point (which input each
gradient goes to, the activation store handed from forward to backward, lse kept out of the
graph), checked on the CPU with the fp64 oracle standing in for the library's calls."""
import numpy as np
import pytest
import torch

import oracle
from global_attention_b200.autograd import zgcm_attention
from global_attention_b200.synth import make_inputs


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def _oracle_ops(store_bytes, seen):
    def fwd(q, k, v, g, gq, gk, *, window, rope_dims, rope_base, eps, scale, saved=None):
        seen["fwd_store"] = saved
        P = oracle.Problem(q, k, v, g, gq, gk, window=window, rope_dims=rope_dims, rope_base=rope_base, eps=eps,
                           scale=scale)
        out, lse = P.forward()
        return torch.from_numpy(out), torch.from_numpy(lse)

    def bwd(q, k, v, g, gq, gk, out, lse, dout, *, window, rope_dims, rope_base, eps, scale, saved=None):
        seen["bwd_store"] = saved
        P = oracle.Problem(q, k, v, g, gq, gk, window=window, rope_dims=rope_dims, rope_base=rope_base, eps=eps,
                           scale=scale)
        return {n: torch.from_numpy(x) for n, x in P.backward(dout).items()}

    def size(B, S, Hq, Hkv, D, rope_dims, window):
        return store_bytes

    return fwd, bwd, size


@pytest.mark.parametrize("store_bytes", [256, 0])
def test_gradients_reach_their_inputs(store_bytes):
    t = make_inputs(2, 40, Hq=4, Hkv=2, D=16, seed=5, with_dout=True)
    names = ("q", "k", "v", "g", "gamma_q", "gamma_k")
    x = {n: t[n].double().requires_grad_(True) for n in names}
    seen = {}
    kw = dict(window=8, rope_dims=8, rope_base=500.0, eps=1e-6)
    out, lse = zgcm_attention(*(x[n] for n in names), return_lse=True, ops=_oracle_ops(store_bytes, seen), **kw)
    assert not lse.requires_grad
    dout = t["dout"].double()
    (out * dout).sum().backward()
    # the store (when the pair applies) is the same tensor in both passes
    if store_bytes:
        assert seen["fwd_store"] is not None and seen["bwd_store"] is seen["fwd_store"]
        assert seen["fwd_store"].numel() == store_bytes
    else:
        assert seen["fwd_store"] is None and seen["bwd_store"] is None
    P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], scale=16 ** -0.5, **kw)
    ref_out, ref_lse = P.forward()
    np.testing.assert_array_equal(out.detach().numpy(), ref_out)
    np.testing.assert_array_equal(lse.numpy(), ref_lse)
    ref = P.backward(dout)
    for n, r in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("gamma_q", "dgamma_q"),
                 ("gamma_k", "dgamma_k")):
        np.testing.assert_array_equal(x[n].grad.numpy(), ref[r], err_msg=n)


@pytest.mark.gpu
@pytest.mark.parametrize("S,W", [(700, 128), (500, 10**6)])
def test_autograd_on_the_gpu_matches_oracle(S, W):
    """zgcm_attention end to end on the B200 (the library's training pair under autograd):
    a loss sum(dout * out) backpropagated to every input equals the oracle's gradients."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.parity_util import assert_bf16_close, assert_dgamma_close
    t = make_inputs(1, S, seed=31 + S, with_dout=True)
    leaves = {n: t[n].cuda().requires_grad_(True) for n in ("q", "k", "v", "g", "gamma_q", "gamma_k")}
    out = zgcm_attention(*(leaves[n] for n in ("q", "k", "v", "g", "gamma_q", "gamma_k")), window=W)
    (out.float() * t["dout"].cuda().float()).sum().backward()
    torch.cuda.synchronize()
    P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], window=W)
    ref_out, _ = P.forward()
    ref = P.backward(t["dout"])
    assert_bf16_close("out", out.detach(), ref_out)
    for n, r in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg")):
        assert_bf16_close(r, leaves[n].grad, ref[r])
    assert_dgamma_close("dgamma_q", leaves["gamma_q"].grad, ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", leaves["gamma_k"].grad, ref["dgamma_k"])
