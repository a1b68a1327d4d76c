"""GPU vs fp64 oracle, element by element, through the C ABI (needs a B200).

Small and ragged shapes are compared in full (every output element); the full-size
workloads of the layer (16K SWA fwd/bwd, 64K global fwd+bwd, 256K SWA and global fwd)
are compared on sampled rows the oracle computes one by one, plus properties that hold
at any size.
"""
import numpy as np
import pytest
import torch

import global_attention_b200 as ga
import oracle
from global_attention_b200.synth import make_inputs, sample_query_rows
from tests.parity_util import (assert_bf16_close, assert_dgamma_close, assert_lse_close, f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ga.load()
    oracle.build()


def _to_dev(t):
    return {k: v.cuda() for k, v in t.items()}


def _gpu_fwd(d, **kw):
    out, lse = ga.zgcm_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], **kw)
    torch.cuda.synchronize()
    # an expired bounded wait leaves outputs unwritten: never compare those
    assert ga.zgcm_attn_device_error() == 0
    return out, lse


def _gpu_bwd(d, out, lse, **kw):
    gr = ga.zgcm_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], out, lse,
                          d["dout"], **kw)
    torch.cuda.synchronize()
    assert ga.zgcm_attn_device_error() == 0
    return gr


def _problem(t, **kw):
    return oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], **kw)


SMALL = [
    # B, S, Hq, Hkv, W, rope_dims, base
    (1, 1024, 32, 8, 128, 42, 1e4),      # the tiny SWA workload of the layer
    (2, 1000, 32, 8, 128, 42, 1e4),      # ragged tail, two sequences
    (1, 129, 32, 8, 128, 42, 1e4),       # one tile + one row
    (1, 1, 32, 8, 128, 42, 1e4),         # single token
    (1, 300, 8, 8, 1, 42, 1e4),          # self-only window, no GQA sharing
    (1, 333, 4, 1, 2, 128, 1e7),         # two-key window, full rotation, 10M base
    (1, 777, 32, 8, 777, 42, 1e4),       # global layer (W = S), ragged
    (1, 500, 16, 4, 10**6, 0, 1e4),      # global, W >> S, no rotation
    (3, 260, 32, 8, 200, 42, 1e4),       # window between one and two tiles
    (2, 45, 4, 1, 128, 42, 1e4),         # strips: one KV head, sequences of 1.4 strips
    (5, 77, 32, 8, 100, 42, 1e4),        # strips: one strip per CTA, every span loaded whole
    (1, 3000, 16, 8, 128, 42, 1e4),      # two query heads per KV head: per-head tcgen05 kernel
]


@pytest.mark.parametrize("B,S,Hq,Hkv,W,R,base", SMALL)
def test_small_full_compare(B, S, Hq, Hkv, W, R, base):
    t = make_inputs(B, S, Hq=Hq, Hkv=Hkv, seed=B * 7 + S + W % 97, with_dout=True)
    kw = dict(window=W, rope_dims=R, rope_base=base)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d, **kw)
    P = _problem(t, **kw)
    ref_out, ref_lse = P.forward()
    assert_bf16_close("out", out, ref_out)
    assert_lse_close("lse", lse, ref_lse)
    gr = _gpu_bwd(d, out, lse, **kw)
    ref = P.backward(t["dout"])
    for n in ("dq", "dk", "dv", "dg"):
        assert_bf16_close(n, gr[n], ref[n])
    assert_dgamma_close("dgamma_q", gr["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", gr["dgamma_k"], ref["dgamma_k"])


@pytest.mark.parametrize("B,S,W", [(1, 1024, 128), (2, 1000, 128), (1, 129, 7), (3, 260, 1), (1, 1, 128),
                                   (2, 384, 100)])
def test_forward_strip_kernel(B, S, W):
    """The strip kernel (windows up to 128, 4 query heads per KV head) matches the oracle."""
    t = make_inputs(B, S, seed=100 + S + W)
    d = _to_dev(t)
    ref_out, ref_lse = _problem(t, window=W).forward()
    assert ga.zgcm_attn_fwd_kernel_name(B, S, 32, 8, 42, W) == "fwd_strip_kernel"
    out, lse = _gpu_fwd(d, window=W)
    assert ga.zgcm_attn_device_error() == 0
    assert_bf16_close("out", out, ref_out)
    assert_lse_close("lse", lse, ref_lse)


# Shapes off the layer's own (42 rotated dims, 4 query heads per KV head): every kernel has a
# second instance for any number of rotated pairs, and the per-head and wide-window kernels
# take any group size (odd ones included).  (B, S, Hq, Hkv, W, rope_dims, forward kernel)
OTHER_SHAPES = [
    (1, 700, 32, 8, 128, 0, "fwd_strip_kernel"),       # no rotation
    (2, 300, 32, 8, 77, 128, "fwd_strip_kernel"),      # every dim rotated
    (1, 520, 32, 8, 128, 64, "fwd_strip_kernel"),
    (1, 650, 24, 8, 128, 42, "fwd_tc_kernel"),         # 3 query heads per KV head
    (2, 260, 16, 2, 100, 126, "fwd_tc_kernel"),        # 8 per KV head
    (1, 300, 8, 8, 1, 2, "fwd_tc_kernel"),             # plain multi-head, window 1
    (1, 900, 24, 8, 900, 42, "fwd_glob_tc_kernel"),    # odd group, global layer
    (2, 400, 8, 8, 300, 2, "fwd_glob_tc_kernel"),      # one query head per KV head
    (1, 333, 40, 8, 10**6, 0, "fwd_glob_tc_kernel"),   # 5 per KV head, no rotation
    (1, 500, 6, 2, 200, 128, "fwd_glob_tc_kernel"),    # 3 per KV head, every dim rotated
]


@pytest.mark.parametrize("B,S,Hq,Hkv,W,R,kname", OTHER_SHAPES)
def test_other_shapes_forward_backward(B, S, Hq, Hkv, W, R, kname):
    """Forward and backward on the shapes above match the oracle, through the kernel named."""
    t = make_inputs(B, S, Hq=Hq, Hkv=Hkv, seed=900 + S + R + W % 1000, with_dout=True)
    kw = dict(window=W, rope_dims=R)
    d = _to_dev(t)
    P = _problem(t, **kw)
    ref_out, ref_lse = P.forward()
    assert ga.zgcm_attn_fwd_kernel_name(B, S, Hq, Hkv, R, W) == kname
    out, lse = _gpu_fwd(d, **kw)
    assert ga.zgcm_attn_device_error() == 0
    assert_bf16_close("out", out, ref_out)
    assert_lse_close("lse", lse, ref_lse)
    gr = _gpu_bwd(d, out, lse, **kw)
    assert ga.zgcm_attn_device_error() == 0
    ref = P.backward(t["dout"])
    for n in ("dq", "dk", "dv", "dg"):
        assert_bf16_close(n, gr[n], ref[n])
    assert_dgamma_close("dgamma_q", gr["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", gr["dgamma_k"], ref["dgamma_k"])
    # the training pair on the same shape: bit-identical to the plain pair
    n = ga.zgcm_attn_saved_size(B, S, Hq, Hkv, rope_dims=R, window=W)
    assert n > 0
    saved = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    out_s, lse_s = _gpu_fwd(d, saved=saved, **kw)
    assert torch.equal(out, out_s) and torch.equal(lse, lse_s)
    gr_s = _gpu_bwd(d, out_s, lse_s, saved=saved, **kw)
    assert ga.zgcm_attn_device_error() == 0
    for name in gr:
        assert torch.equal(gr[name], gr_s[name]), name


@pytest.mark.parametrize("gq_all,spike,B,S,W", [
    (1.0, 20.0, 1, 1000, 128),     # two large gamma_q entries: bound far above the limit
    (1.9, None, 2, 700, 128),      # gamma 1.9 everywhere: bound just under the limit (59.2)
    (2.0, None, 1, 333, 37),       # gamma 2.0 everywhere: just over it (65.6)
])
def test_forward_score_bound_fallback(gq_all, spike, B, S, W):
    """The sliding-window forward takes its exponentials' reference from a bound on every
    score, |scale| log2(e) D max|gamma_q| max|gamma_k|, when that bound is at most 60, and
    from each row's maximum otherwise.  Both sides of the limit, and a bound far above it,
    match the oracle."""
    t = make_inputs(B, S, seed=500 + S + W)
    gq = torch.full((128,), gq_all, dtype=torch.float32)
    if spike is not None:
        gq[:2] = spike
    t["gamma_q"] = gq
    t["gamma_k"] = torch.full((128,), gq_all, dtype=torch.float32)
    d = _to_dev(t)
    ref_out, ref_lse = _problem(t, window=W).forward()
    assert ga.zgcm_attn_fwd_kernel_name(B, S, 32, 8, 42, W) == "fwd_strip_kernel"
    out, lse = _gpu_fwd(d, window=W)
    assert ga.zgcm_attn_device_error() == 0
    assert_bf16_close("out", out, ref_out)
    assert_lse_close("lse", lse, ref_lse)


@pytest.mark.parametrize("B,S,W", [(1, 777, 777), (2, 1000, 10**6), (1, 129, 129), (1, 1, 4096),
                                   (3, 260, 200), (1, 1300, 300), (2, 640, 129), (1, 2048, 2048)])
def test_forward_wide_window_kernel(B, S, W):
    """Windows wider than one key tile (the global layer W >= S among them) run the tcgen05
    wide-window forward; it matches the oracle."""
    t = make_inputs(B, S, seed=300 + S + W % 1000)
    d = _to_dev(t)
    ref_out, ref_lse = _problem(t, window=W).forward()
    assert ga.zgcm_attn_fwd_kernel_name(B, S, 32, 8, 42, W) == "fwd_glob_tc_kernel"
    out, lse = _gpu_fwd(d, window=W)
    assert ga.zgcm_attn_device_error() == 0
    assert_bf16_close("out", out, ref_out)
    assert_lse_close("lse", lse, ref_lse)
    # the same call through the plain C entry (scratch from the stream-ordered pool)
    import ctypes
    lib = ga.load()
    out2, lse2 = torch.empty_like(out), torch.empty_like(lse)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())
    st = lib.zgcm_attn_fwd(vp(d["q"]), vp(d["k"]), vp(d["v"]), vp(d["g"]), vp(d["gamma_q"]), vp(d["gamma_k"]),
                           B, S, 32, 8, 128, 42, 10000.0, W, 1, 1e-6, 128 ** -0.5, vp(out2), vp(lse2),
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == 0
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("B,S,W", [(1, 1024, 128), (2, 1000, 128), (1, 129, 7), (3, 260, 1), (1, 1, 128),
                                   (2, 384, 100)])
def test_backward_sliding_kernels(B, S, W):
    """The tcgen05 backward pair of windows up to 128 matches the oracle's gradients."""
    t = make_inputs(B, S, seed=200 + S + W, with_dout=True)
    d = _to_dev(t)
    ref = _problem(t, window=W).backward(t["dout"])
    assert ga.zgcm_attn_bwd_kernel_names(S, W)[:5] == ["bwd_gate_kernel", "bwd_prep_kv_kernel", "bwd_prep_q_kernel",
                                                        "bwd_q_tc_kernel", "bwd_kv_tc_kernel"]
    out, lse = _gpu_fwd(d, window=W)
    gr = _gpu_bwd(d, out, lse, window=W)
    assert ga.zgcm_attn_device_error() == 0
    for n in ("dq", "dk", "dv", "dg"):
        assert_bf16_close(n, gr[n], ref[n])
    assert_dgamma_close("dgamma_q", gr["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", gr["dgamma_k"], ref["dgamma_k"])


@pytest.mark.parametrize("B,S,W", [(1, 777, 777), (2, 1000, 10**6), (1, 129, 129), (1, 1, 4096),
                                   (3, 260, 200), (1, 1300, 300), (2, 640, 129), (1, 2048, 2048)])
def test_backward_wide_window_kernels(B, S, W):
    """Windows wider than one key tile (the global layer among them) run the tcgen05
    wide-window backward (tile bounds, query-major dq sweep, key-major dk/dv sweep); every
    gradient matches the oracle."""
    t = make_inputs(B, S, seed=400 + S + W % 1000, with_dout=True)
    d = _to_dev(t)
    ref = _problem(t, window=W).backward(t["dout"])
    assert ga.zgcm_attn_bwd_kernel_names(S, W) == [
        "bwd_gate_kernel", "bwd_prep_kv_kernel", "bwd_prep_q_kernel", "bwd_tile_stats_kernel",
        "bwd_q_glob_kernel", "bwd_kv_tc_kernel", "dgamma_reduce_kernel(k)", "dgamma_reduce_kernel(q)"]
    out, lse = _gpu_fwd(d, window=W)
    gr = _gpu_bwd(d, out, lse, window=W)
    assert ga.zgcm_attn_device_error() == 0
    for n in ("dq", "dk", "dv", "dg"):
        assert_bf16_close(n, gr[n], ref[n])
    assert_dgamma_close("dgamma_q", gr["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", gr["dgamma_k"], ref["dgamma_k"])


def _decode_run(t, W, C, offsets=None, rope_dims=42):
    """Feed each sequence of t token by token through zgcm_attn_decode; sequence b starts
    offsets[b] calls late (before that it replays its token 0 at position 0, which rewrites the
    same cache slot with the same values).  Returns out [T, B, Hq, D], lse [T, B, Hq], pos [T, B]."""
    B, S, Hq, D = t["q"].shape
    Hkv = t["k"].shape[2]
    offsets = offsets or [0] * B
    d = _to_dev(t)
    kc = torch.zeros((B, C, Hkv, D), dtype=torch.float16, device="cuda")
    vc = torch.zeros((B, C, Hkv, D), dtype=torch.bfloat16, device="cuda")
    outs, lses, poss = [], [], []
    ar = torch.arange(B, device="cuda")
    for call in range(S + max(offsets)):
        pos = torch.tensor([min(max(call - o, 0), S - 1) for o in offsets], dtype=torch.int32, device="cuda")
        pl = pos.long()
        o, l = ga.zgcm_attn_decode(d["q"][ar, pl].contiguous(), d["k"][ar, pl].contiguous(),
                                   d["v"][ar, pl].contiguous(), d["g"][ar, pl].contiguous(),
                                   d["gamma_q"], d["gamma_k"], pos, kc, vc, window=W, rope_dims=rope_dims)
        outs.append(o.clone()); lses.append(l.clone()); poss.append(pos.cpu())
    torch.cuda.synchronize()
    return torch.stack(outs), torch.stack(lses), torch.stack(poss)


@pytest.mark.parametrize("B,S,W", [(1, 1024, 128), (2, 1000, 128), (1, 129, 7), (3, 260, 1), (1, 1, 128),
                                   (1, 777, 777), (2, 640, 129), (1, 1300, 300)])
def test_saved_activations_bit_identical(B, S, W):
    """zgcm_attn_fwd(saved=...) then zgcm_attn_bwd(saved=...) gives exactly the results of the
    plain pair: the store holds the q~, k~ and inverse RMS values the backward's preparation
    would form (the store starts out filled with garbage)."""
    t = make_inputs(B, S, seed=700 + S + W % 1000, with_dout=True)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d, window=W)
    gr = _gpu_bwd(d, out, lse, window=W)
    n = ga.zgcm_attn_saved_size(B, S, 32, 8, window=W)
    assert n > 0
    saved = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    out_s, lse_s = _gpu_fwd(d, window=W, saved=saved)
    assert torch.equal(out, out_s) and torch.equal(lse, lse_s)
    gr_s = _gpu_bwd(d, out_s, lse_s, window=W, saved=saved)
    assert ga.zgcm_attn_device_error() == 0
    for name in gr:
        assert torch.equal(gr[name], gr_s[name]), name


@pytest.mark.parametrize("B,S,W,C", [(2, 300, 128, 128),     # sliding layer: a ring of W slots
                                     (1, 700, 700, 768),     # global layer: every token kept, 2 splits
                                     (3, 200, 50, 64),       # ring larger than the window
                                     (2, 1100, 10**6, 1100)])  # global, 3 splits of 512 keys
def test_decode_matches_forward_rows(B, S, W, C):
    """Decoding a sequence token by token gives, at every step, the forward's row for that
    position (the oracle's), through the layer's sliding ring cache or its growing one."""
    t = make_inputs(B, S, seed=500 + S + W % 997)
    out, lse, pos = _decode_run(t, W, C)
    ref_out, ref_lse = _problem(t, window=W).forward()
    # call c decodes position c of every sequence
    got = f64(out).transpose(1, 0, 2, 3)          # [B, S, Hq, D]
    assert_bf16_close("decode out", got, ref_out)
    assert_lse_close("decode lse", f64(lse).transpose(1, 2, 0), ref_lse)
    assert ga.zgcm_attn_device_error() == 0


def test_decode_ragged_positions_and_short_cache():
    B, S, W = 3, 160, 128
    t = make_inputs(B, S, seed=77)
    offsets = [0, 7, 33]
    out, lse, pos = _decode_run(t, W, W, offsets=offsets)
    ref_out, ref_lse = _problem(t, window=W).forward()
    for b, o in enumerate(offsets):
        calls = np.arange(o, o + S)
        got = f64(out[calls, b])                  # positions 0..S-1 of sequence b
        assert_bf16_close(f"decode out[{b}]", got, ref_out[b])
    # a window longer than the cache: rows past the cache get NaN, earlier ones are exact
    out2, lse2, _ = _decode_run(make_inputs(1, 100, seed=3), 80, 64)
    o2 = f64(out2)
    assert np.isnan(o2[64:]).all() and np.isfinite(o2[:64]).all()


def test_bounded_wait_expires_and_is_reported():
    """A wait nothing satisfies gives up after its bound, the kernel returns, the host reads
    ZGCM_ERR_TIMEOUT (once), and the context still computes correct results."""
    import time
    assert ga.zgcm_attn_device_error() == 0
    t0 = time.perf_counter()
    assert ga.zgcm_attn_selftest_expired_wait() == 0
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert ga.zgcm_attn_device_error() == -6      # ZGCM_ERR_TIMEOUT
    assert ga.zgcm_attn_device_error() == 0       # read and cleared
    assert waited < 60.0
    t = make_inputs(1, 256, seed=12)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d)
    ref_out, _ = _problem(t).forward()
    assert_bf16_close("out after the expired wait", out, ref_out)


def test_halo_rows_match_whole_sequence():
    """The premise of the sliding layer's sequence sharding on the CUDA kernels: the rows of
    a chunk computed from [the previous W - 1 key/value rows; the chunk], with zero query and
    gate rows under the halo and positions numbered from 0, equal the same rows of the
    whole-sequence call (outputs, lse, dq, dg, and dk, dv of the rows no later chunk sees)."""
    B, L, W, R = 2, 640, 128, 3
    t = make_inputs(B, R * L, seed=61, with_dout=True)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d, window=W)
    gr = _gpu_bwd(d, out, lse, window=W)
    h = W - 1
    for r in range(1, R):
        a, s0, e = r * L - h, r * L, (r + 1) * L
        zq = torch.zeros_like(d["q"][:, :h])
        ext = dict(q=torch.cat([zq, d["q"][:, s0:e]], 1).contiguous(), k=d["k"][:, a:e].contiguous(),
                   v=d["v"][:, a:e].contiguous(), g=torch.cat([zq, d["g"][:, s0:e]], 1).contiguous(),
                   gamma_q=d["gamma_q"], gamma_k=d["gamma_k"],
                   dout=torch.cat([zq, d["dout"][:, s0:e]], 1).contiguous())
        o, l = _gpu_fwd(ext, window=W)
        assert_bf16_close(f"out[{r}]", o[:, h:], f64(out)[:, s0:e])
        assert_lse_close(f"lse[{r}]", l[:, :, h:], f64(lse)[:, :, s0:e])
        g2 = _gpu_bwd(ext, o, l, window=W)
        for n in ("dq", "dg"):
            assert_bf16_close(f"{n}[{r}]", g2[n][:, h:], f64(gr[n])[:, s0:e])
        for n in ("dk", "dv"):  # rows the next chunk's queries do not see
            assert_bf16_close(f"{n}[{r}]", g2[n][:, h:L], f64(gr[n])[:, s0:e - h])


def test_training_step_in_a_cuda_graph():
    """The calls are stream-ordered, never synchronise and allocate nothing when given their
    buffers, so a training step (the pair that keeps activations) captures into a CUDA graph;
    a replay gives exactly the eager results, also after new inputs are copied in."""
    B, S, W = 2, 1000, 128
    d = _to_dev(make_inputs(B, S, seed=71, with_dout=True))
    sv = torch.empty(ga.zgcm_attn_saved_size(B, S, 32, 8, window=W), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ga.zgcm_attn_bwd_workspace_size(B, S, 32, 8, 128, W), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])
    lse = torch.empty((B, 32, S), dtype=torch.float32, device="cuda")
    grads = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]), dv=torch.empty_like(d["v"]),
                 dg=torch.empty_like(d["g"]), dgamma_q=torch.empty(128, device="cuda"),
                 dgamma_k=torch.empty(128, device="cuda"))

    def step():
        ga.zgcm_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], window=W, out=out,
                         lse=lse, saved=sv)
        ga.zgcm_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], out, lse, d["dout"],
                         window=W, grads=grads, workspace=ws, saved=sv)

    def results():
        return [out.clone(), lse.clone()] + [grads[n].clone() for n in sorted(grads)]

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # eager, outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = results()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for x in [out, lse] + list(grads.values()):
        x.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert ga.zgcm_attn_device_error() == 0
    for a, b in zip(eager, results()):
        assert torch.equal(a, b)
    # new inputs in the same buffers: the replay follows them
    d2 = _to_dev(make_inputs(B, S, seed=72, with_dout=True))
    for n in d:
        d[n].copy_(d2[n])
    graph.replay()
    torch.cuda.synchronize()
    replayed = results()
    step()
    torch.cuda.synchronize()
    assert ga.zgcm_attn_device_error() == 0
    for a, b in zip(replayed, results()):
        assert torch.equal(a, b)
    del graph


def test_empty_problem():
    for B, S in ((0, 16), (2, 0)):
        t = make_inputs(max(B, 1), max(S, 1), with_dout=True)
        d = {k: (v[:B, :S].contiguous().cuda() if v.dim() == 4 else v.cuda()) for k, v in t.items()}
        out, lse = _gpu_fwd(d)
        assert out.numel() == 0 and lse.numel() == 0
        gr = _gpu_bwd(d, out, lse)
        assert torch.all(gr["dgamma_q"] == 0) and torch.all(gr["dgamma_k"] == 0)


def test_gate_limits_and_nan():
    t = make_inputs(1, 256, seed=3, with_dout=True)
    g = t["g"].clone()
    g[0, :, 0, :] = float("inf")
    g[0, :, 1, :] = float("-inf")
    g[0, 17, 2, 5] = float("nan")
    t["g"] = g
    d = _to_dev(t)
    out, lse = _gpu_fwd(d)
    ref_out, _ = _problem(t).forward()
    o = f64(out)
    assert np.isnan(o[0, 17, 2, 5]) and np.isnan(ref_out[0, 17, 2, 5])
    mask = np.ones(o.shape, bool)
    mask[0, 17, 2, 5] = False
    assert_bf16_close("out(g=+-inf)", o[mask], ref_out[mask])
    assert np.all(o[0, :, 1, :] == 0.0)


def test_timed_backward_matches_untimed():
    """zgcm_attn_bwd_timed (events around each kernel) does the same work."""
    t = make_inputs(1, 640, seed=9, with_dout=True)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d)
    names = ga.zgcm_attn_bwd_kernel_names(640, 128)
    assert len(names) >= 3
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in names]
    g1 = _gpu_bwd(d, out, lse)
    g2 = ga.zgcm_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["gamma_q"], d["gamma_k"], out, lse, d["dout"],
                          kernel_events=ev)
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dg", "dgamma_q", "dgamma_k"):
        assert torch.equal(g1[n], g2[n]), n
    assert all(a.elapsed_time(b) >= 0.0 for a, b in ev)


def test_forward_bitwise_repeatable():
    t = make_inputs(2, 2048, seed=5)
    d = _to_dev(t)
    o1, l1 = _gpu_fwd(d)
    o2, l2 = _gpu_fwd(d)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------------ full-size workloads

def _sampled_fwd_bwd(B, S, W, n_random, k_rows, check_bwd=True, seed=0, edge=256, saved_pair=False):
    t = make_inputs(B, S, seed=seed, with_dout=check_bwd)
    d = _to_dev(t)
    out, lse = _gpu_fwd(d, window=W)
    gr = _gpu_bwd(d, out, lse, window=W) if check_bwd else None
    if saved_pair:
        # the training pair the benchmark times gives exactly these results at this size
        sv = torch.empty(ga.zgcm_attn_saved_size(B, S, 32, 8, window=W), dtype=torch.uint8, device="cuda")
        out_s, lse_s = _gpu_fwd(d, window=W, saved=sv)
        assert torch.equal(out, out_s) and torch.equal(lse, lse_s)
        gr_s = _gpu_bwd(d, out_s, lse_s, window=W, saved=sv)
        for name in gr:
            assert torch.equal(gr[name], gr_s[name]), name
        del sv, out_s, lse_s, gr_s
    P = _problem(t, window=W)
    rows = sample_query_rows(B, S, n_random=n_random, edge=edge, seed=seed)
    b, i = rows // S, rows % S
    ref_out, ref_lse = P.forward(rows)
    assert_bf16_close("out[rows]", f64(out)[b, i], ref_out)
    assert_lse_close("lse[rows]", f64(lse)[b, :, i], ref_lse)
    if not check_bwd:
        return
    dq, dg = P.backward_qrows(t["dout"], rows)
    assert_bf16_close("dq[rows]", f64(gr["dq"])[b, i], dq)
    assert_bf16_close("dg[rows]", f64(gr["dg"])[b, i], dg)
    kb, ki = k_rows // S, k_rows % S
    dk, dv = P.backward_krows(t["dout"], k_rows)
    assert_bf16_close("dk[rows]", f64(gr["dk"])[kb, ki], dk)
    assert_bf16_close("dv[rows]", f64(gr["dv"])[kb, ki], dv)
    # any-size properties: sum_j dv_j = sum_{h in group, i} dout_i * sigmoid(g_i)
    G = t["q"].shape[2] // t["k"].shape[2]
    dA = (d["dout"].double() * torch.sigmoid(d["g"].double()))
    rhs = dA.view(B, S, -1, G, 128).sum(dim=(1, 3))
    lhs = gr["dv"].double().sum(dim=1)
    assert_bf16_close("sum_j dv", lhs, rhs, atol=2e-2 * float(rhs.abs().max()) + 2e-2)
    # gamma_q . dgamma_q = gamma_k . dgamma_k (scores are invariant to q_hat*c, k_hat/c).
    # Each side sums B*S*H rows of gradient terms that carry the per-element error the
    # bf16 bound allows (rel-RMS 5e-3) and largely cancel, so the two sums are compared
    # to 2e-2 of their size.
    a = float((gr["dgamma_q"].double() * d["gamma_q"].double()).sum())
    c = float((gr["dgamma_k"].double() * d["gamma_k"].double()).sum())
    assert abs(a - c) <= 2e-2 * max(abs(a), abs(c)) + 1e-3, (a, c)


def test_swa_16k_forward_backward():
    """B=4, S=16384, W=128: forward and backward on sampled rows + properties."""
    B, S = 4, 16384
    rng = np.random.default_rng(1)
    k_rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(S * B - 64, S * B),
                                       rng.integers(0, B * S, 128)]))
    _sampled_fwd_bwd(B, S, 128, n_random=512, k_rows=k_rows, saved_pair=True)


def test_global_64k_forward_backward():
    """Global layer: B=1, S=65536, W=S, sampled rows + properties.  A query row late in the
    sequence costs the oracle O(S); a key row j needs the softmax statistics of every query
    row after it, O(S^2) for an early key, so only the last keys are affordable here.  The
    heaviest key tiles of the global backward (those that accumulate over the most query
    blocks) are compared in test_global_8k_heaviest_key_tiles."""
    S = 65536
    k_rows = np.arange(S - 48, S)
    _sampled_fwd_bwd(1, S, S, n_random=96, k_rows=k_rows, edge=16, saved_pair=True)


def test_global_8k_heaviest_key_tiles():
    """Global layer at S=8192: dk and dv of the first three key tiles (rows 0..383), the units
    of the key-major kernel that accumulate over the most query blocks (64, 63, 62 blocks of
    128 queries x 4 heads) and run first on its heaviest-first schedule; plus sampled query rows."""
    S = 8192
    k_rows = np.arange(0, 384)
    _sampled_fwd_bwd(1, S, S, n_random=64, k_rows=k_rows, edge=32, saved_pair=True, seed=3)


def test_swa_16k_every_element():
    """The headline workload compared in full: B=4, S=16384, W=128, every element of out, lse,
    dq, dk, dv, dg and both d_gamma against the oracle's full forward and backward, computed by
    the training pair the benchmark times (the forward keeping its activations)."""
    import psutil
    if psutil.virtual_memory().available < 48e9:
        pytest.skip("needs ~30 GB of host RAM for the fp64 oracle arrays at B=4, S=16384")
    B, S, W = 4, 16384, 128
    t = make_inputs(B, S, seed=0, with_dout=True)
    d = _to_dev(t)
    sv = torch.empty(ga.zgcm_attn_saved_size(B, S, 32, 8, window=W), dtype=torch.uint8, device="cuda")
    out, lse = _gpu_fwd(d, window=W, saved=sv)
    gr = _gpu_bwd(d, out, lse, window=W, saved=sv)
    got = {"out": out.cpu(), "lse": lse.cpu(), **{n: x.cpu() for n, x in gr.items()}}
    del d, sv, out, lse, gr
    P = _problem(t, window=W)
    ref_out, ref_lse = P.forward()
    for b in range(B):
        assert_bf16_close(f"out[b={b}]", got["out"][b], ref_out[b])
    assert_lse_close("lse", got["lse"], ref_lse)
    del ref_out, ref_lse
    ref = P.backward(t["dout"])
    for n in ("dq", "dk", "dv", "dg"):
        for b in range(B):
            assert_bf16_close(f"{n}[b={b}]", got[n][b], ref[n][b])
        # and over the whole tensor (rel-RMS of the full gradient)
        assert_bf16_close(n, got[n], ref[n])
    assert_dgamma_close("dgamma_q", got["dgamma_q"], ref["dgamma_q"])
    assert_dgamma_close("dgamma_k", got["dgamma_k"], ref["dgamma_k"])


def test_256k_swa_and_global_forward():
    import psutil
    if psutil.virtual_memory().available < 96e9:
        pytest.skip("needs ~40 GB of host RAM for the fp64 oracle arrays at S=262144")
    S = 262144
    t = make_inputs(1, S, seed=0)
    d = _to_dev(t)
    P = _problem(t, window=128)
    rows = sample_query_rows(1, S, n_random=256, edge=256, seed=0)
    out, lse = _gpu_fwd(d, window=128)
    ro, rl = P.forward(rows)
    assert_bf16_close("swa out[rows]", f64(out)[0, rows], ro)
    assert_lse_close("swa lse[rows]", f64(lse)[0, :, rows], rl)
    del out, lse
    out, lse = _gpu_fwd(d, window=S)
    grows = np.unique(np.concatenate([np.arange(0, 64), np.arange(S - 3, S),
                                      np.random.default_rng(2).integers(0, S, 5)]))
    P.set_window(S)
    ro, rl = P.forward(grows)
    assert_bf16_close("global out[rows]", f64(out)[0, grows], ro)
    assert_lse_close("global lse[rows]", f64(lse)[0, :, grows], rl)
