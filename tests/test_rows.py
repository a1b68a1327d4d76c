"""Query rows at the end of a longer key sequence (zgcm_attn_fwd_rows / zgcm_attn_bwd_rows):
one shard of a sequence-sharded global layer, computed on the B200 with the first-query-row
offset and compared with the fp64 oracle's rows for that shard (the oracle runs the whole
sequence; the shard's output and query gradients are its rows from q_off on, its key
gradients and d_gamma those of a backward whose output gradient is zero before q_off)."""
import numpy as np
import pytest
import torch

import global_attention_b200 as ga
import oracle
from global_attention_b200.synth import make_inputs
from tests.parity_util import assert_bf16_close, assert_dgamma_close, assert_lse_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ga.load()
    oracle.build()


# (B, S key rows, Sq query rows, window): the global layer with the shard in the middle of a
# query block's worth of rows and a ragged last block; a wide window whose first key tile
# (the one of key q_off - W + 1) is past the sequence start, so the key rows before it get
# no query at all; the last block alone; every row (the plain entry points)
CASES = [(2, 1024, 384, 10**6), (1, 1300, 788, 300), (1, 1000, 232, 10**6), (1, 640, 640, 640),
         (1, 896, 128, 200)]


@pytest.mark.parametrize("B,S,Sq,W", CASES)
def test_query_rows_match_oracle_shard(B, S, Sq, W):
    q_off = S - Sq
    t = make_inputs(B, S, seed=1200 + S + Sq, with_dout=True)
    zero = t["dout"].clone()
    zero[:, :q_off] = 0  # the other shards' output gradients: not this shard's business
    P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], window=W)
    ref_out, ref_lse = P.forward()
    ref = P.backward(zero)
    d = {n: x.cuda() for n, x in t.items()}
    shard = {n: d[n][:, q_off:].contiguous() for n in ("q", "g", "dout")}
    out, lse = ga.zgcm_attn_fwd_rows(shard["q"], d["k"], d["v"], shard["g"], d["gamma_q"], d["gamma_k"], window=W)
    gr = ga.zgcm_attn_bwd_rows(shard["q"], d["k"], d["v"], shard["g"], d["gamma_q"], d["gamma_k"], out, lse,
                               shard["dout"], window=W)
    torch.cuda.synchronize()
    assert ga.zgcm_attn_device_error() == 0
    assert_bf16_close("out", out, ref_out[:, q_off:])
    assert_lse_close("lse", lse, ref_lse[:, :, q_off:])
    for n in ("dq", "dg"):
        assert_bf16_close(n, gr[n], ref[n][:, q_off:])
    for n in ("dk", "dv"):
        assert_bf16_close(n, gr[n], ref[n])
    assert_dgamma_close("dgamma_q", gr["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", gr["dgamma_k"], ref["dgamma_k"])
    if W == 300:  # keys 0..127 are before every query's window: exactly zero
        assert torch.all(gr["dk"][:, :128] == 0) and torch.all(gr["dv"][:, :128] == 0)


def test_no_query_rows():
    """Sq = 0: nothing to attend; the backward leaves zero key gradients and d_gamma."""
    t = make_inputs(1, 256, seed=5, with_dout=True)
    d = {n: x.cuda() for n, x in t.items()}
    q0 = d["q"][:, :0].contiguous()
    out, lse = ga.zgcm_attn_fwd_rows(q0, d["k"], d["v"], q0, d["gamma_q"], d["gamma_k"], window=256)
    assert out.shape == (1, 0, 32, 128) and lse.shape == (1, 32, 0)
    grads = dict(dq=torch.empty_like(q0), dk=torch.full_like(d["k"], 7.0), dv=torch.full_like(d["v"], 7.0),
                 dg=torch.empty_like(q0), dgamma_q=torch.full((128,), 7.0, device="cuda"),
                 dgamma_k=torch.full((128,), 7.0, device="cuda"))
    ga.zgcm_attn_bwd_rows(q0, d["k"], d["v"], q0, d["gamma_q"], d["gamma_k"], out, lse, q0, window=256, grads=grads)
    torch.cuda.synchronize()
    for n in ("dk", "dv", "dgamma_q", "dgamma_k"):
        assert torch.all(grads[n] == 0), n
