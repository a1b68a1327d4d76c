"""The backward for callers that cannot allocate device memory.

A process that has reserved the GPU's memory for its own pool, or a plugin that is given
no allocator, cannot hand zgcm_attn_bwd a workspace; zgcm_attn_bwd_noalloc uses the
library's fixed per-device scratch array instead.  Its results must match the workspace
entry point's, call after call (the scratch keeps the previous call's contents).

This file is collected last on purpose, and passes both on its own in a fresh process and
after the other tests.
"""
import ctypes

import pytest
import torch

import global_attention_b200 as ga
from global_attention_b200.synth import make_inputs
from tests.parity_util import assert_bf16_close, assert_dgamma_close

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg")


def _noalloc_via_cabi(d, out, lse, grads, window):
    """Call zgcm_attn_bwd_noalloc through the C ABI with raw pointers."""
    lib = ga.load()
    B, S, Hq, D = d["q"].shape
    Hkv = d["k"].shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.zgcm_attn_bwd_noalloc(
        p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]), p(d["gamma_q"]), p(d["gamma_k"]), p(out), p(lse), p(d["dout"]),
        B, S, Hq, Hkv, D, 42, 10000.0, window, 1, 1e-6, 1.0 / D ** 0.5,
        p(grads["dq"]), p(grads["dk"]), p(grads["dv"]), p(grads["dg"]), p(grads["dgamma_q"]), p(grads["dgamma_k"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ga.load()


def test_noalloc_matches_workspace_backward_on_consecutive_calls():
    # the last call is the largest problem the 64 MiB array takes at 32/8 heads and W = 128
    for call, (B, S, W, seed) in enumerate(((1, 1000, 128, 11), (2, 700, 128, 12), (1, 3117, 128, 13))):
        t = make_inputs(B, S, seed=seed, with_dout=True)
        d = {k: v.cuda() for k, v in t.items()}
        out, lse = ga.zgcm_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], window=W)
        ref = ga.zgcm_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], out, lse, d["dout"],
                               window=W)
        got = {n: torch.full_like(x, float("nan")) for n, x in ref.items()}
        st = _noalloc_via_cabi(d, out, lse, got, W)
        torch.cuda.synchronize()
        assert st == 0, ga.zgcm_status_string(st)
        for n in GRADS:
            assert_bf16_close(f"call {call} {n}", got[n], ref[n])
        assert_dgamma_close(f"call {call} dgamma_q", got["dgamma_q"], ref["dgamma_q"])
        assert_dgamma_close(f"call {call} dgamma_k", got["dgamma_k"], ref["dgamma_k"])


def test_noalloc_rejects_problems_beyond_its_scratch():
    null = ctypes.c_void_p(0)
    st = ga.load().zgcm_attn_bwd_noalloc(*([null] * 9), 4, 16384, 32, 8, 128, 42, 10000.0, 128, 1, 1e-6,
                                         0.0883883, *([null] * 7))
    assert st == -7 and "TOO_LARGE" in ga.zgcm_status_string(st)
