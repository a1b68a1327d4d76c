"""C-ABI library: loads, exports every declared symbol, and rejects bad arguments on the
host before any launch.  CPU only: no call here reaches a kernel."""
import ctypes
import os
import re

import pytest

import global_attention_b200 as ga
from global_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return ga.load()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(zgcm_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert {"zgcm_attn_fwd", "zgcm_attn_bwd", "zgcm_attn_bwd_workspace_size",
            "zgcm_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        getattr(lib, n)  # resolves through dlsym


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert ga.zgcm_status_string(st).startswith("ZGCM_")
    assert "unknown" in ga.zgcm_status_string(12345)


# fake, 256-byte aligned, never dereferenced: every call below fails validation first
P = 0x7F0000000000
ARGS = dict(B=1, S=64, Hq=32, Hkv=8, D=128, rope_dims=42, rope_base=10000.0, window=128, causal=1,
            eps=1e-6, scale=0.0883883)


def _fwd(lib, ptrs=None, **kw):
    a = dict(ARGS, **kw)
    p = ptrs or [P + 256 * i for i in range(8)]
    vp = ctypes.c_void_p
    return lib.zgcm_attn_fwd(*(vp(x) for x in p[:6]), a["B"], a["S"], a["Hq"], a["Hkv"], a["D"],
                             a["rope_dims"], a["rope_base"], a["window"], a["causal"], a["eps"],
                             a["scale"], vp(p[6]), vp(p[7]), None)


def _bwd(lib, ws_bytes, ws=P + 256 * 40, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(15)]
    return lib.zgcm_attn_bwd(*p[:9], a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                             a["rope_base"], a["window"], a["causal"], a["eps"], a["scale"],
                             *p[9:15], vp(ws), ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(D=64), -2), (dict(causal=0), -2), (dict(causal=2), -1), (dict(Hq=30), -1),
    (dict(window=0), -1), (dict(rope_dims=41), -1), (dict(rope_dims=130), -1),
    (dict(eps=-1.0), -1), (dict(scale=0.0), -1), (dict(scale=float("nan")), -1),
    (dict(B=-1), -1), (dict(S=-5), -1), (dict(Hkv=0), -1), (dict(rope_base=0.0), -1),
])
def test_fwd_rejects_bad_arguments(lib, kw, status):
    assert _fwd(lib, **kw) == status


def test_fwd_pointer_checks(lib):
    good = [P + 256 * i for i in range(8)]
    for i in range(8):
        p = list(good); p[i] = 0
        assert _fwd(lib, ptrs=p) == -1
        p = list(good); p[i] = good[i] + 8
        assert _fwd(lib, ptrs=p) == -3


def test_bwd_workspace_checks(lib):
    need = lib.zgcm_attn_bwd_workspace_size(1, 64, 32, 8, 128, 128)
    assert need > 0
    assert _bwd(lib, need - 1) == -4
    assert _bwd(lib, need, ws=0) == -4
    assert _bwd(lib, need, ws=P + 256 * 40 + 16) == -3
    assert _bwd(lib, need, D=100) == -2


def test_workspace_size_query(lib):
    ws = lambda *a: lib.zgcm_attn_bwd_workspace_size(*a)
    assert ws(0, 64, 32, 8, 128, 128) == 0
    assert ws(1, 0, 32, 8, 128, 128) == 0
    assert ws(1, 64, 32, 8, 64, 128) == 0   # unsupported D -> 0
    assert ws(4, 16384, 32, 8, 128, 128) > ws(1, 16384, 32, 8, 128, 128) > ws(1, 1024, 32, 8, 128, 128)
    assert ws(1, 1024, 32, 8, 128, 128) % 256 == 0


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(ga, "_lib", None)
    monkeypatch.setattr(ga, "LIB_PATH", "/nonexistent/libzgcm_attn.so")
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        ga.load()


def _fwd_ws(lib, ws, ws_bytes, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(8)]
    return lib.zgcm_attn_fwd_ws(*p[:6], a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                a["rope_base"], a["window"], a["causal"], a["eps"], a["scale"],
                                p[6], p[7], vp(ws), ws_bytes, None)


def test_fwd_workspace_size_query(lib):
    ws = lambda *a: lib.zgcm_attn_fwd_workspace_size(*a)
    # the sliding layer (W <= 128, 4 query heads per KV head) needs none: the strip kernel
    # normalises its key chunks in shared memory, so zgcm_attn_fwd allocates nothing there
    for B, S, W in ((4, 16384, 128), (1, 1024, 7), (1, 1, 128), (2, 1000, 1)):
        assert ws(B, S, 32, 8, 128, 42, W) == 0
    # wider windows (the global layer among them) read the fp16 normalised keys, [B, S, Hkv, D],
    # prepared once per key tile
    for B, S, W in ((1, 65536, 65536), (2, 1000, 300), (1, 1, 10**6), (3, 777, 129)):
        n = B * S * 8 * 128 * 2
        assert ws(B, S, 32, 8, 128, 42, W) == (n + 255) // 256 * 256
    # other group sizes of the sliding layer take the per-head tcgen05 kernel, which reads them too
    assert ws(1, 1024, 16, 8, 128, 42, 128) == (1024 * 8 * 256 + 255) // 256 * 256
    # any number of rotated dims and any group size: the same rule
    assert ws(1, 1024, 32, 8, 128, 0, 1024) == (1024 * 8 * 256 + 255) // 256 * 256
    assert ws(1, 1024, 32, 8, 128, 128, 128) == 0
    assert ws(1, 1024, 24, 8, 128, 42, 1024) == (1024 * 8 * 256 + 255) // 256 * 256
    assert ws(1, 1024, 8, 8, 128, 0, 64) == (1024 * 8 * 256 + 255) // 256 * 256
    # invalid or empty -> 0
    assert ws(1, 1024, 32, 8, 64, 42, 1024) == 0
    assert ws(0, 1024, 32, 8, 128, 42, 1024) == 0
    assert ws(1, 1024, 30, 8, 128, 42, 1024) == 0


def test_fwd_ws_checks(lib):
    need = lib.zgcm_attn_fwd_workspace_size(1, 640, 32, 8, 128, 42, 640)
    assert need > 0
    assert _fwd_ws(lib, P + 256 * 40, need - 1, S=640, window=640) == -4
    assert _fwd_ws(lib, 0, need, S=640, window=640) == -4
    assert _fwd_ws(lib, P + 256 * 40 + 16, need, S=640, window=640) == -3
    assert _fwd_ws(lib, P + 256 * 40, need, S=640, window=640, D=96) == -2
    assert _fwd_ws(lib, P + 256 * 40, need, S=640, window=0) == -1


def test_saved_size_query(lib):
    sz = lambda *a: lib.zgcm_attn_saved_size(*a)
    al = lambda x: (x + 255) // 256 * 256
    # q~ fp16, q inverse RMS, k~ fp16, k inverse RMS, each 256-byte aligned
    for B, S, W in ((4, 16384, 128), (1, 1000, 7), (2, 777, 10**6), (1, 1, 128), (3, 260, 129)):
        rows, krows = B * S * 32, B * S * 8
        assert sz(B, S, 32, 8, 128, 42, W) == al(rows * 256) + al(rows * 4) + al(krows * 256) + al(krows * 4)
    # every shape: no rotation, all dims rotated, an odd group size with a wide window
    for Hq, R, W in ((32, 0, 128), (32, 128, 1024), (24, 42, 1024)):
        rows, krows = 1024 * Hq, 1024 * 8
        assert sz(1, 1024, Hq, 8, 128, R, W) == al(rows * 256) + al(rows * 4) + al(krows * 256) + al(krows * 4)
    assert sz(0, 1024, 32, 8, 128, 42, 128) == 0      # empty
    assert sz(1, 1024, 32, 8, 64, 42, 128) == 0       # invalid


def _fwd_save(lib, saved, saved_bytes, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(8)]
    return lib.zgcm_attn_fwd_save(*p[:6], a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                  a["rope_base"], a["window"], a["causal"], a["eps"], a["scale"],
                                  p[6], p[7], vp(saved), saved_bytes, None)


def _bwd_saved(lib, ws_bytes, saved, saved_bytes, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(15)]
    return lib.zgcm_attn_bwd_saved(*p[:9], a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                   a["rope_base"], a["window"], a["causal"], a["eps"], a["scale"], *p[9:15],
                                   vp(P + 256 * 40), ws_bytes, vp(saved), saved_bytes, None, None, 0)


def test_saved_pair_checks(lib):
    need = lib.zgcm_attn_saved_size(1, 64, 32, 8, 128, 42, 128)
    assert need > 0
    store = P + 2 ** 30
    assert _fwd_save(lib, store, need - 1) == -4          # too small
    assert _fwd_save(lib, 0, need) == -4                  # missing
    assert _fwd_save(lib, store + 16, need) == -3         # not 256-byte aligned
    assert _fwd_save(lib, store, need, D=96) == -2        # head size other than 128
    assert _fwd_save(lib, store, need, window=0) == -1
    ws = lib.zgcm_attn_bwd_workspace_size(1, 64, 32, 8, 128, 128)
    assert _bwd_saved(lib, ws, 0, need) == -1             # the store is required
    assert _bwd_saved(lib, ws, store, need - 1) == -4
    assert _bwd_saved(lib, ws, store + 16, need) == -3
    assert _bwd_saved(lib, ws - 1, store, need) == -4     # the workspace is checked as before
    assert _bwd_saved(lib, ws, store, need, D=96) == -2
    names = ga.zgcm_attn_bwd_kernel_names(16384, 128, saved=True)
    assert names[:4] == ["bwd_gate_kernel", "bwd_prep_v_kernel", "bwd_q_tc_kernel", "bwd_kv_tc_kernel"]
    assert "bwd_prep_q_kernel" not in ga.zgcm_attn_bwd_kernel_names(4096, 4096, saved=True)


def _dec(lib, ws_bytes, ptrs=None, ws=P + 256 * 40, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = ptrs or [P + 256 * i for i in range(11)]
    return lib.zgcm_attn_decode(*(vp(x) for x in p[:7]), a["B"], a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                a["rope_base"], a["window"], a["eps"], a["scale"], vp(p[7]), vp(p[8]),
                                a.get("cache_len", 128), vp(p[9]), vp(p[10]), vp(ws), ws_bytes, None)


def test_decode_checks(lib):
    need = lib.zgcm_attn_decode_workspace_size(1, 32, 128, 128)
    # per (sequence, head): 4 records (one per warp) per split of up to 512 keys, each max, sum,
    # 2 pad and 128 partial outputs
    assert need == 1 * 32 * 1 * 4 * (4 + 128) * 4
    assert lib.zgcm_attn_decode_workspace_size(2, 32, 10**6, 65536) == 2 * 32 * 128 * 4 * 132 * 4
    assert lib.zgcm_attn_decode_workspace_size(2, 32, 300, 65536) == 2 * 32 * 1 * 4 * 132 * 4
    assert lib.zgcm_attn_decode_workspace_size(0, 32, 128, 128) == 0
    assert _dec(lib, need - 1) == -4
    assert _dec(lib, need, ws=0) == -4
    assert _dec(lib, need, cache_len=0) == -1
    assert _dec(lib, need, D=64) == -2
    assert _dec(lib, need, window=0) == -1
    good = [P + 256 * i for i in range(11)]
    for i in range(11):
        p = list(good); p[i] = 0
        assert _dec(lib, need, ptrs=p) == -1
        p = list(good); p[i] = good[i] + 4
        assert _dec(lib, need, ptrs=p) == -3


def _noalloc(lib, B, S, W=128):
    null = [ctypes.c_void_p(0)] * 16
    return lib.zgcm_attn_bwd_noalloc(*null[:9], B, S, 32, 8, 128, 42, 10000.0, W, 1, 1e-6, 0.0883883,
                                     *null[9:16])


def test_noalloc_size_bound(lib):
    """The no-allocation backward takes every problem whose workspace fits its 64 MiB array and
    rejects the rest with ZGCM_ERR_TOO_LARGE (-7) before looking at anything else; at 32/8
    heads and a window of 128 the bound is B*S = 3117 tokens (the figure the header states)."""
    lim = 64 << 20
    ws = lambda B, S: lib.zgcm_attn_bwd_workspace_size(B, S, 32, 8, 128, 128)
    s_ok = max(S for S in range(3000, 3300) if ws(1, S) <= lim)
    assert s_ok == 3117
    # accepted by the size check: the null tensor pointers are what it then rejects (-1)
    assert _noalloc(lib, 1, s_ok) == -1
    assert _noalloc(lib, 1, s_ok + 1) == -7
    assert _noalloc(lib, 4, 16384) == -7


def test_noalloc_binding_checks_before_any_launch(monkeypatch):
    """The Python wrapper checks dtype, rank, layout and device of every tensor before it
    reaches the C entry point: a float32 or a transposed q never gets to a kernel."""
    import torch
    from global_attention_b200.synth import make_inputs
    reached = []

    class NoLib:
        def __getattr__(self, name):
            reached.append(name)
            raise AssertionError(f"reached the library ({name})")

    monkeypatch.setattr(ga, "load", lambda: NoLib())
    t = make_inputs(1, 8, with_dout=True)
    lse = torch.zeros((1, 32, 8), dtype=torch.float32)
    args = dict(q=t["q"], k=t["k"], v=t["v"], g=t["g"], gamma_q=t["gamma_q"], gamma_k=t["gamma_k"],
                out=t["q"].clone(), lse=lse, dout=t["dout"])
    for bad in (dict(q=t["q"].float()), dict(q=t["q"].transpose(1, 2)), dict(lse=lse.double()),
                dict(gamma_k=t["gamma_k"].half()), dict(dout=t["dout"][:, :, :, :64])):
        with pytest.raises(TypeError, match="contiguous"):
            ga.zgcm_attn_bwd_noalloc(**dict(args, **bad))
    with pytest.raises(TypeError, match="CUDA"):
        ga.zgcm_attn_bwd_noalloc(**args)
    assert not reached


def _fwd_rows(lib, ws, ws_bytes, Sq, S, window, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(8)]
    return lib.zgcm_attn_fwd_rows(*p[:6], a["B"], Sq, S, a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                  a["rope_base"], window, a["causal"], a["eps"], a["scale"], p[6], p[7],
                                  vp(ws), ws_bytes, None)


def _bwd_rows(lib, ws, ws_bytes, Sq, S, window, **kw):
    a = dict(ARGS, **kw)
    vp = ctypes.c_void_p
    p = [vp(P + 256 * i) for i in range(15)]
    return lib.zgcm_attn_bwd_rows(*p[:9], a["B"], Sq, S, a["Hq"], a["Hkv"], a["D"], a["rope_dims"],
                                  a["rope_base"], window, a["causal"], a["eps"], a["scale"], *p[9:15],
                                  vp(ws), ws_bytes, None)


def test_query_rows_checks(lib):
    """Query rows at the end of the key rows: Sq <= S, and a first query row off position 0
    only on a 128-row boundary with a window wider than 128; the workspace is the one of the
    whole key sequence.  Every call here fails validation before any launch."""
    need = lib.zgcm_attn_fwd_workspace_size(1, 640, 32, 8, 128, 42, 640)
    ws = P + 256 * 40
    for fn, n in ((_fwd_rows, need), (_bwd_rows, lib.zgcm_attn_bwd_workspace_size(1, 640, 32, 8, 128, 640))):
        assert fn(lib, ws, n, Sq=641, S=640, window=640) == -1     # more query rows than keys
        assert fn(lib, ws, n, Sq=-1, S=640, window=640) == -1
        assert fn(lib, ws, n, Sq=600, S=640, window=640) == -2     # first query row off a 128 boundary
        assert fn(lib, ws, n, Sq=512, S=640, window=128) == -2     # a window of at most 128
        assert fn(lib, ws, n, Sq=512, S=640, window=640, D=96) == -2
        assert fn(lib, 0, n, Sq=512, S=640, window=640) == -4      # workspace missing
        assert fn(lib, ws, n - 1, Sq=512, S=640, window=640) == -4
        assert fn(lib, ws + 16, n, Sq=512, S=640, window=640) == -3


def test_muon_checks(lib):
    """Muon calls reject bad dimensions, pointers, alignment and workspace before any launch."""
    vp = ctypes.c_void_p
    lib.zgcm_muon_workspace_size.restype = ctypes.c_size_t
    ws = lib.zgcm_muon_workspace_size
    assert ws(4096, 11008) == ws(11008, 4096) > 0
    for m, n in ((7, 16), (16, 12), (0, 8), (8, -8)):
        assert ws(m, n) == 0
    need = ws(64, 128)
    f = ctypes.c_float
    step = lambda W, G, M, m, n, steps, wsp, wsb: lib.zgcm_muon_step(
        vp(W), vp(G), vp(M), m, n, f(2e-4), f(0.1), f(0.9), steps, f(1.5), f(-0.5), f(0.0), f(1e-7), vp(wsp), wsb,
        None)
    orth = lambda G, O, m, n, steps, wsp, wsb: lib.zgcm_muon_orthogonalize(
        vp(G), vp(O), m, n, steps, f(1.5), f(-0.5), f(0.0), f(1e-7), vp(wsp), wsb, None)
    W, G, M, O, S = P, P + 2 ** 20, P + 2 ** 21, P + 2 ** 22, P + 2 ** 23
    assert step(W, G, M, 64, 12, 5, S, need) == -1          # n not a multiple of 8
    assert step(W, G, M, 64, 128, 101, S, need) == -1       # too many steps
    assert step(0, G, M, 64, 128, 5, S, need) == -1
    assert step(W + 4, G, M, 64, 128, 5, S, need) == -3
    assert step(W, G, M, 64, 128, 5, S, need - 1) == -4
    assert step(W, G, M, 64, 128, 5, S + 16, need) == -3
    assert orth(G, O, 64, 124, 5, S, need) == -1
    assert orth(G, 0, 64, 128, 5, S, need) == -1
    assert orth(G, O, 64, 128, 5, 0, need) == -4
    gemm = lambda A, B, D, C, M_, N_, K_, kn: lib.zgcm_muon_gemm(vp(A), vp(B), vp(D), vp(C), M_, N_, K_, f(1.0),
                                                                 f(0.0), kn, None)
    assert gemm(G, G, 0, O, 64, 12, 64, 0) == -1            # N not a multiple of 8
    assert gemm(G, G, 0, O, 64, 64, 60, 0) == -1            # K neither
    assert gemm(G, G, 0, O, 64, 64, 64, 2) == -1            # layout flag
    assert gemm(G, G, 0, 0, 64, 64, 64, 0) == -1
    assert gemm(G + 8, G, 0, O, 64, 64, 64, 0) == -3


def test_proj_checks(lib):
    """Projection calls reject shapes the tiles cannot split and bad pointers before any launch."""
    vp = ctypes.c_void_p
    x, w, q, k, v, g = (P + (1 << 22) * i for i in range(6))
    fwd = lambda T, dm, Hq, Hkv, D, ptrs=(x, w, q, k, v, g): lib.zgcm_proj_qkvg_fwd(
        vp(ptrs[0]), vp(ptrs[1]), T, dm, Hq, Hkv, D, *(vp(t) for t in ptrs[2:]), None)
    assert fwd(0, 512, 4, 2, 128) == -1                      # no tokens
    assert fwd(64, 500, 4, 2, 128) == -1                     # d_model not a multiple of 256
    assert fwd(64, 512, 3, 1, 64) == -1                      # Hkv * D = 64
    assert fwd(64, 512, 4, 2, 128, (x, w, q, 0, v, g)) == -1
    assert fwd(64, 512, 4, 2, 128, (x, w + 8, q, k, v, g)) == -3
    out = lambda T, din, dm, y=q: lib.zgcm_proj_out_fwd(vp(x), vp(w), T, din, dm, vp(y), None)
    assert out(64, 512, 300) == -1
    assert out(64, 512, 512, 0) == -1
    bwd = lambda da: lib.zgcm_proj_out_bwd(vp(x), vp(w), vp(q), 64, 512, 512, vp(da), vp(k), None)
    assert bwd(v + 4) == -3


def test_bindings_check_shapes_before_any_launch(monkeypatch):
    """The library sees pointers and sizes only, so each Python wrapper checks that every tensor
    has the shape the sizes it passes imply (and dtype, layout and one CUDA device) before the
    C entry point: a tensor shorter than that would be read or written past its end.  Each bad
    call below fails on the CPU with a shape error; the consistent one gets as far as the
    device check."""
    import torch
    from global_attention_b200.synth import make_inputs
    reached = []

    class NoLib:
        def __getattr__(self, name):
            reached.append(name)
            raise AssertionError(f"reached the library ({name})")

    monkeypatch.setattr(ga, "load", lambda: NoLib())
    t = make_inputs(1, 16, with_dout=True)
    q, k, v, g, gq, gk, do = (t[n] for n in ("q", "k", "v", "g", "gamma_q", "gamma_k", "dout"))
    lse = torch.zeros((1, 32, 16), dtype=torch.float32)
    bf = dict(dtype=torch.bfloat16)

    def shape_error(fn, *a, **kw):
        with pytest.raises(TypeError, match="shape|sequence length|must be \\[|inner dimensions|four tensors"):
            fn(*a, **kw)

    def device_error(fn, *a, **kw):
        with pytest.raises(TypeError, match="CUDA"):
            fn(*a, **kw)

    lay = dict(q=q, k=k, v=v, g=g, gamma_q=gq, gamma_k=gk)
    # forward
    for bad in (dict(v=v[:, :8].contiguous()), dict(g=g[:, :, :16].contiguous()), dict(gamma_q=gq[:64].contiguous()),
                dict(k=k[:, :8].contiguous(), v=v[:, :8].contiguous()),
                dict(k=torch.zeros((2, 16, 8, 128), **bf), v=torch.zeros((2, 16, 8, 128), **bf))):
        shape_error(ga.zgcm_attn_fwd, **dict(lay, **bad))
    shape_error(ga.zgcm_attn_fwd, **lay, out=torch.zeros((1, 8, 32, 128), **bf))
    shape_error(ga.zgcm_attn_fwd, **lay, lse=torch.zeros((1, 32, 8)))
    device_error(ga.zgcm_attn_fwd, **lay)
    # backward (plain, query rows, no allocation)
    bw = dict(lay, out=q.clone(), lse=lse, dout=do)
    grads = dict(dq=torch.zeros_like(q), dk=torch.zeros_like(k), dv=torch.zeros_like(v), dg=torch.zeros_like(g),
                 dgamma_q=torch.zeros(128), dgamma_k=torch.zeros(128))
    for fn in (ga.zgcm_attn_bwd, ga.zgcm_attn_bwd_noalloc):
        shape_error(fn, **dict(bw, lse=torch.zeros((1, 32, 8))))
        shape_error(fn, **dict(bw, out=torch.zeros((1, 8, 32, 128), **bf)))
        shape_error(fn, **dict(bw, dout=torch.zeros((1, 16, 16, 128), **bf)))
        shape_error(fn, **bw, grads=dict(grads, dk=torch.zeros((1, 16, 4, 128), **bf)))
        shape_error(fn, **bw, grads=dict(grads, dgamma_k=torch.zeros(64)))
        device_error(fn, **bw, grads=grads)
    rows = dict(lay, q=q[:, 8:].contiguous(), g=g[:, 8:].contiguous())
    shape_error(ga.zgcm_attn_fwd_rows, **dict(rows, k=torch.zeros((1, 16, 8, 64), **bf)), window=4096)
    shape_error(ga.zgcm_attn_fwd_rows, **rows, lse=lse, window=4096)
    device_error(ga.zgcm_attn_fwd_rows, **rows, window=4096)
    rows_b = dict(rows, out=rows["q"].clone(), lse=torch.zeros((1, 32, 8)), dout=do[:, 8:].contiguous())
    shape_error(ga.zgcm_attn_bwd_rows, **dict(rows_b, lse=lse), window=4096)
    device_error(ga.zgcm_attn_bwd_rows, **rows_b, window=4096)
    # decode
    dec = dict(q=q[:, 0].contiguous(), k=k[:, 0].contiguous(), v=v[:, 0].contiguous(), g=g[:, 0].contiguous(),
               gamma_q=gq, gamma_k=gk, pos=torch.zeros(1, dtype=torch.int32),
               k_cache=torch.zeros((1, 128, 8, 128), dtype=torch.float16), v_cache=torch.zeros((1, 128, 8, 128), **bf))
    shape_error(ga.zgcm_attn_decode, **dict(dec, v_cache=torch.zeros((1, 64, 8, 128), **bf)))
    shape_error(ga.zgcm_attn_decode, **dict(dec, pos=torch.zeros(2, dtype=torch.int32)))
    shape_error(ga.zgcm_attn_decode, **dict(dec, g=torch.zeros((1, 16, 128), **bf)))
    device_error(ga.zgcm_attn_decode, **dec)
    # Muon
    W, G, M = torch.zeros((64, 96)), torch.zeros((64, 96), **bf), torch.zeros((64, 96))
    shape_error(ga.zgcm_muon_step, W, G[:32].contiguous(), M)
    shape_error(ga.zgcm_muon_step, W, G, torch.zeros((96, 64)))
    device_error(ga.zgcm_muon_step, W, G, M)
    shape_error(ga.zgcm_muon_orthogonalize, G, out=torch.zeros((96, 64), **bf))
    device_error(ga.zgcm_muon_orthogonalize, G)
    A, Bm = torch.zeros((64, 32), **bf), torch.zeros((48, 32), **bf)
    shape_error(ga.zgcm_muon_gemm, A, Bm, out=torch.zeros((64, 32), **bf))
    shape_error(ga.zgcm_muon_gemm, A, Bm, D=torch.zeros((48, 64), **bf))
    shape_error(ga.zgcm_muon_gemm, A, Bm, b_kn=True)
    device_error(ga.zgcm_muon_gemm, A, Bm)
    # projections (Hq = 4, Hkv = 2, D = 128: W_qkvg has 12 x 128 rows)
    x, w = torch.zeros((8, 256), **bf), torch.zeros((12 * 128, 256), **bf)
    pj = dict(Hq=4, Hkv=2, D=128)
    shape_error(ga.zgcm_proj_qkvg_fwd, x, w[:-128].contiguous(), **pj)
    shape_error(ga.zgcm_proj_qkvg_fwd, x, w, out=(torch.zeros((8, 512), **bf),) * 3, **pj)
    shape_error(ga.zgcm_proj_qkvg_fwd, x, w, out=tuple(torch.zeros((8, 256), **bf) for _ in range(4)), **pj)
    device_error(ga.zgcm_proj_qkvg_fwd, x, w, **pj)
    dq_, dk_ = torch.zeros((8, 512), **bf), torch.zeros((8, 256), **bf)
    shape_error(ga.zgcm_proj_qkvg_bwd, x, w, dq_, dk_, dk_, dk_, **pj)
    shape_error(ga.zgcm_proj_qkvg_bwd, x, w, dq_, dk_, dk_, dq_, dx=torch.zeros((8, 128), **bf), **pj)
    device_error(ga.zgcm_proj_qkvg_bwd, x, w, dq_, dk_, dk_, dq_, **pj)
    a_, wo = torch.zeros((8, 512), **bf), torch.zeros((256, 512), **bf)
    shape_error(ga.zgcm_proj_out_fwd, a_, torch.zeros((256, 384), **bf))
    shape_error(ga.zgcm_proj_out_fwd, a_, wo, out=torch.zeros((8, 512), **bf))
    device_error(ga.zgcm_proj_out_fwd, a_, wo)
    shape_error(ga.zgcm_proj_out_bwd, a_, wo, torch.zeros((8, 512), **bf))
    shape_error(ga.zgcm_proj_out_bwd, a_, wo, torch.zeros((8, 256), **bf), dw=torch.zeros((512, 256), **bf))
    device_error(ga.zgcm_proj_out_bwd, a_, wo, torch.zeros((8, 256), **bf))
    assert not reached
