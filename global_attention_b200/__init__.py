"""ZGCM-1 gated window-attention layer on B200: Python binding of the C ABI.

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libzgcm_attn.so`` (built in-tree by ``python -m global_attention_b200.build``).  There is
no CPU fallback; if the library is missing, loading fails loudly.

The functions carry the C names (include/zgcm_attn.h) and take torch CUDA tensors:

    out, lse = zgcm_attn_fwd(q, k, v, g, gamma_q, gamma_k, window=128)
    grads = zgcm_attn_bwd(q, k, v, g, gamma_q, gamma_k, out, lse, dout, window=128)

q, g, dout: bf16 [B,S,Hq,128]; k, v: bf16 [B,S,Hkv,128]; gamma_*: fp32 [128].
"""
from __future__ import annotations

import ctypes
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzgcm_attn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "zgcm_attn.h")

ZGCM_OK = 0
_lib = None


class ZgcmError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {zgcm_status_string(status)} ({status})")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libzgcm_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m global_attention_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i, d, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float
        lib.zgcm_status_string.argtypes = [i]
        lib.zgcm_status_string.restype = ctypes.c_char_p
        lib.zgcm_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, d, i, i, f, f, vp, vp, vp]
        lib.zgcm_attn_fwd.restype = i
        lib.zgcm_attn_fwd_ws.argtypes = lib.zgcm_attn_fwd.argtypes[:-1] + [vp, ctypes.c_size_t, vp]
        lib.zgcm_attn_fwd_ws.restype = i
        lib.zgcm_attn_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i]
        lib.zgcm_attn_fwd_workspace_size.restype = ctypes.c_size_t
        lib.zgcm_attn_decode.argtypes = [vp] * 7 + [i] * 5 + [d, i, f, f, vp, vp, i, vp, vp, vp,
                                                              ctypes.c_size_t, vp]
        lib.zgcm_attn_decode.restype = i
        lib.zgcm_attn_decode_workspace_size.argtypes = [i, i, i, i]
        lib.zgcm_attn_decode_workspace_size.restype = ctypes.c_size_t
        lib.zgcm_attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
        lib.zgcm_attn_bwd_workspace_size.restype = ctypes.c_size_t
        lib.zgcm_attn_bwd.argtypes = ([vp] * 9 + [i] * 6 + [d, i, i, f, f] + [vp] * 7 +
                                      [ctypes.c_size_t, vp])
        lib.zgcm_attn_bwd.restype = i
        lib.zgcm_attn_bwd_timed.argtypes = lib.zgcm_attn_bwd.argtypes + [ctypes.POINTER(vp), i]
        lib.zgcm_attn_bwd_timed.restype = i
        lib.zgcm_attn_bwd_kernel_name.argtypes = [i, i, i, i]
        lib.zgcm_attn_bwd_kernel_name.restype = ctypes.c_char_p
        lib.zgcm_attn_bwd_saved_kernel_name.argtypes = [i, i, i, i]
        lib.zgcm_attn_bwd_saved_kernel_name.restype = ctypes.c_char_p
        lib.zgcm_attn_saved_size.argtypes = [i, i, i, i, i, i, i]
        lib.zgcm_attn_saved_size.restype = ctypes.c_size_t
        lib.zgcm_attn_fwd_save.argtypes = lib.zgcm_attn_fwd_ws.argtypes
        lib.zgcm_attn_fwd_save.restype = i
        lib.zgcm_attn_bwd_saved.argtypes = (lib.zgcm_attn_bwd.argtypes[:-1] + [vp, ctypes.c_size_t, vp,
                                                                               ctypes.POINTER(vp), i])
        lib.zgcm_attn_bwd_saved.restype = i
        lib.zgcm_attn_fwd_kernel_name.argtypes = [i, i, i, i, i, i]
        lib.zgcm_attn_fwd_kernel_name.restype = ctypes.c_char_p
        lib.zgcm_attn_selftest_expired_wait.argtypes = [vp]
        lib.zgcm_attn_selftest_expired_wait.restype = i
        lib.zgcm_attn_device_error.argtypes = []
        lib.zgcm_attn_device_error.restype = i
        lib.zgcm_attn_bwd_noalloc.argtypes = [vp] * 9 + [i] * 6 + [d, i, i, f, f] + [vp] * 7
        lib.zgcm_attn_bwd_noalloc.restype = i
        lib.zgcm_attn_fwd_rows.argtypes = [vp] * 6 + [i] * 7 + [d, i, i, f, f] + [vp, vp, vp, ctypes.c_size_t, vp]
        lib.zgcm_attn_fwd_rows.restype = i
        lib.zgcm_attn_bwd_rows.argtypes = [vp] * 9 + [i] * 7 + [d, i, i, f, f] + [vp] * 7 + [ctypes.c_size_t, vp]
        lib.zgcm_attn_bwd_rows.restype = i
        lib.zgcm_muon_workspace_size.argtypes = [i, i]
        lib.zgcm_muon_workspace_size.restype = ctypes.c_size_t
        lib.zgcm_muon_step.argtypes = [vp, vp, vp, i, i, f, f, f, i, f, f, f, f, vp, ctypes.c_size_t, vp]
        lib.zgcm_muon_step.restype = i
        lib.zgcm_muon_orthogonalize.argtypes = [vp, vp, i, i, i, f, f, f, f, vp, ctypes.c_size_t, vp]
        lib.zgcm_muon_orthogonalize.restype = i
        lib.zgcm_muon_gemm.argtypes = [vp, vp, vp, vp, i, i, i, f, f, i, vp]
        lib.zgcm_muon_gemm.restype = i
        lib.zgcm_proj_qkvg_fwd.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, vp, vp]
        lib.zgcm_proj_qkvg_fwd.restype = i
        lib.zgcm_proj_qkvg_bwd.argtypes = [vp] * 6 + [i] * 5 + [vp, vp, vp]
        lib.zgcm_proj_qkvg_bwd.restype = i
        lib.zgcm_proj_out_fwd.argtypes = [vp, vp, i, i, i, vp, vp]
        lib.zgcm_proj_out_fwd.restype = i
        lib.zgcm_proj_out_bwd.argtypes = [vp, vp, vp, i, i, i, vp, vp, vp]
        lib.zgcm_proj_out_bwd.restype = i
        _lib = lib
    return _lib


def zgcm_status_string(status: int) -> str:
    return load().zgcm_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, ndim, cuda=True):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} tensor of rank {ndim}")
    if cuda and not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")


def _need(t, name, dtype, shape):
    """t: a contiguous tensor of `dtype` and exactly `shape` (no device check)."""
    _check(t, name, dtype, len(shape), cuda=False)
    if tuple(t.shape) != tuple(shape):
        raise TypeError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")


def _one_device(*named):
    """Every tensor given (None skipped) is a CUDA tensor on the device of the first one.
    The library sees pointers and sizes only, so the shapes are checked before this, and
    before any launch: a tensor smaller than the sizes passed would be read or written past
    its end."""
    ts = [(n, t) for n, t in named if t is not None]
    for n, t in ts:
        if not t.is_cuda:
            raise TypeError(f"{n} must be a CUDA tensor")
    n0, t0 = ts[0]
    for n, t in ts:
        if t.device != t0.device:
            raise TypeError(f"{n} must be on the device of {n0} ({t0.device})")


def _layer_shapes(q, k, v, g, gamma_q, gamma_k, rows=False):
    """(B, Sq, S, Hq, Hkv, D) of a layer call: q, g [B,Sq,Hq,D] bf16, k, v [B,S,Hkv,D] bf16,
    gamma_q, gamma_k [D] fp32; Sq = S unless `rows` (query rows at the end of the keys)."""
    import torch
    _check(q, "q", torch.bfloat16, 4, cuda=False)
    _check(k, "k", torch.bfloat16, 4, cuda=False)
    B, Sq, Hq, D = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != D:
        raise TypeError(f"k must be [B, S, Hkv, D] with q's B = {B} and D = {D}, not {tuple(k.shape)}")
    if not rows and S != Sq:
        raise TypeError(f"q and k must have one sequence length ({Sq} != {S})")
    _need(v, "v", torch.bfloat16, k.shape)
    _need(g, "g", torch.bfloat16, q.shape)
    _need(gamma_q, "gamma_q", torch.float32, (D,))
    _need(gamma_k, "gamma_k", torch.float32, (D,))
    return B, Sq, S, Hq, Hkv, D


def _check_fwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, workspace, saved=None, rows=False):
    """Dtype, layout and shape of every forward tensor, then their device, before any launch."""
    import torch
    B, Sq, S, Hq, Hkv, D = _layer_shapes(q, k, v, g, gamma_q, gamma_k, rows)
    if out is not None:
        _need(out, "out", torch.bfloat16, q.shape)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, Sq))
    for n, t in (("workspace", workspace), ("saved", saved)):
        if t is not None:
            _check(t, n, torch.uint8, 1, cuda=False)
    _one_device(("q", q), ("k", k), ("v", v), ("g", g), ("gamma_q", gamma_q), ("gamma_k", gamma_k),
                ("out", out), ("lse", lse), ("workspace", workspace), ("saved", saved))
    return B, Sq, S, Hq, Hkv, D


def _check_bwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, dout, grads, workspace=None, saved=None,
                    rows=False):
    """Dtype, layout and shape of every backward tensor, then their device, before any launch."""
    import torch
    B, Sq, S, Hq, Hkv, D = _layer_shapes(q, k, v, g, gamma_q, gamma_k, rows)
    _need(out, "out", torch.bfloat16, q.shape)
    _need(dout, "dout", torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (B, Hq, Sq))
    gl = []
    if grads is not None:
        for n, ref in (("dq", q), ("dk", k), ("dv", v), ("dg", g)):
            _need(grads[n], n, torch.bfloat16, ref.shape)
        for n in ("dgamma_q", "dgamma_k"):
            _need(grads[n], n, torch.float32, (D,))
        gl = [(n, grads[n]) for n in ("dq", "dk", "dv", "dg", "dgamma_q", "dgamma_k")]
    for n, t in (("workspace", workspace), ("saved", saved)):
        if t is not None:
            _check(t, n, torch.uint8, 1, cuda=False)
    _one_device(("q", q), ("k", k), ("v", v), ("g", g), ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("out", out),
                ("lse", lse), ("dout", dout), *gl, ("workspace", workspace), ("saved", saved))
    return B, Sq, S, Hq, Hkv, D


def zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D=128, rope_dims=42, window=128) -> int:
    """Bytes of device scratch the forward needs (0 for windows up to 128)."""
    return int(load().zgcm_attn_fwd_workspace_size(int(B), int(S), int(Hq), int(Hkv), int(D), int(rope_dims),
                                                   int(window)))


def zgcm_attn_saved_size(B, S, Hq, Hkv, D=128, rope_dims=42, window=128) -> int:
    """Bytes of the activation store zgcm_attn_fwd(saved=...) fills for the backward (0 for an
    empty problem)."""
    return int(load().zgcm_attn_saved_size(int(B), int(S), int(Hq), int(Hkv), int(D), int(rope_dims),
                                           int(window)))


def zgcm_attn_fwd(q, k, v, g, gamma_q, gamma_k, *, rope_dims=42, rope_base=10000.0, window=128,
                  causal=1, eps=1e-6, scale=None, out=None, lse=None, workspace=None, saved=None, stream=None):
    """Gated window-attention forward.  Returns (out bf16 [B,S,Hq,D], lse fp32 [B,Hq,S]).
    `workspace`: a uint8 device tensor of at least zgcm_attn_fwd_workspace_size bytes, or None
    to allocate it here when the configuration needs one.  `saved`: a uint8 device tensor of
    zgcm_attn_saved_size bytes (zgcm_attn_fwd_save; then no workspace is used) that keeps the
    activations zgcm_attn_bwd(saved=...) reads."""
    import torch
    B, S, _, Hq, Hkv, D = _check_fwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, workspace, saved)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    if saved is not None:
        st = load().zgcm_attn_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
                                       B, S, Hq, Hkv, D, int(rope_dims), float(rope_base), int(window),
                                       int(causal), float(eps), float(scale), _ptr(out), _ptr(lse),
                                       _ptr(saved), saved.numel(), _stream(stream))
        if st != ZGCM_OK:
            raise ZgcmError(st, "zgcm_attn_fwd_save")
        return out, lse
    need = zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D, rope_dims, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    st = load().zgcm_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
                                 B, S, Hq, Hkv, D, int(rope_dims), float(rope_base), int(window),
                                 int(causal), float(eps), float(scale), _ptr(out), _ptr(lse),
                                 ws_ptr, ws_bytes, _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_fwd")
    return out, lse


def zgcm_attn_decode_workspace_size(B, Hq, window, cache_len) -> int:
    """Bytes of workspace zgcm_attn_decode needs."""
    return int(load().zgcm_attn_decode_workspace_size(int(B), int(Hq), int(window), int(cache_len)))


def zgcm_attn_decode(q, k, v, g, gamma_q, gamma_k, pos, k_cache, v_cache, *, rope_dims=42,
                     rope_base=10000.0, window=128, eps=1e-6, scale=None, out=None, lse=None,
                     workspace=None, stream=None):
    """One decode step: q, g [B,Hq,D] and k, v [B,Hkv,D] bf16 (the new token of each sequence),
    pos int32 [B] (its position), k_cache fp16 / v_cache bf16 [B,C,Hkv,D] (updated in place).
    Returns (out bf16 [B,Hq,D], lse fp32 [B,Hq])."""
    import torch
    _check(q, "q", torch.bfloat16, 3, cuda=False)
    _check(k, "k", torch.bfloat16, 3, cuda=False)
    _check(k_cache, "k_cache", torch.float16, 4, cuda=False)
    B, Hq, D = q.shape
    Hkv, C = k.shape[1], k_cache.shape[1]
    _need(g, "g", torch.bfloat16, (B, Hq, D))
    _need(k, "k", torch.bfloat16, (B, Hkv, D))
    _need(v, "v", torch.bfloat16, (B, Hkv, D))
    _need(gamma_q, "gamma_q", torch.float32, (D,))
    _need(gamma_k, "gamma_k", torch.float32, (D,))
    _need(pos, "pos", torch.int32, (B,))
    _need(k_cache, "k_cache", torch.float16, (B, C, Hkv, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, C, Hkv, D))
    if out is not None:
        _need(out, "out", torch.bfloat16, (B, Hq, D))
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq))
    if workspace is not None:
        _check(workspace, "workspace", torch.uint8, 1, cuda=False)
    _one_device(("q", q), ("k", k), ("v", v), ("g", g), ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("pos", pos),
                ("k_cache", k_cache), ("v_cache", v_cache), ("out", out), ("lse", lse), ("workspace", workspace))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = zgcm_attn_decode_workspace_size(B, Hq, window, C)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = load().zgcm_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k), _ptr(pos),
                                 B, Hq, Hkv, D, int(rope_dims), float(rope_base), int(window), float(eps),
                                 float(scale), _ptr(k_cache), _ptr(v_cache), C, _ptr(out), _ptr(lse),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_decode")
    return out, lse


def zgcm_attn_bwd_workspace_size(B, S, Hq, Hkv, D=128, window=128) -> int:
    return int(load().zgcm_attn_bwd_workspace_size(int(B), int(S), int(Hq), int(Hkv), int(D), int(window)))


def zgcm_attn_fwd_kernel_name(B, S, Hq, Hkv, rope_dims=42, window=128) -> str:
    """Name of the kernel zgcm_attn_fwd launches for this configuration."""
    return load().zgcm_attn_fwd_kernel_name(int(B), int(S), int(Hq), int(Hkv), int(rope_dims),
                                            int(window)).decode()


def zgcm_attn_selftest_expired_wait(stream=None) -> int:
    """Launch the bounded-wait self-test (a wait that expires); see the C header."""
    return int(load().zgcm_attn_selftest_expired_wait(_stream(stream)))


def zgcm_attn_device_error() -> int:
    """ZGCM_OK, or ZGCM_ERR_TIMEOUT if a bounded device wait expired since the last call."""
    return int(load().zgcm_attn_device_error())


def zgcm_attn_bwd_kernel_names(S, window, rope_dims=42, saved=False):
    """Names of the kernels zgcm_attn_bwd launches (with `saved`: zgcm_attn_bwd_saved), in order."""
    names, i = [], 0
    query = load().zgcm_attn_bwd_saved_kernel_name if saved else load().zgcm_attn_bwd_kernel_name
    while True:
        n = query(i, int(S), int(rope_dims), int(window))
        if n is None:
            return names
        names.append(n.decode())
        i += 1


def zgcm_attn_bwd(q, k, v, g, gamma_q, gamma_k, out, lse, dout, *, rope_dims=42, rope_base=10000.0,
                  window=128, causal=1, eps=1e-6, scale=None, grads=None, workspace=None, saved=None,
                  stream=None, kernel_events=None):
    """Gated window-attention backward.  Returns dict dq, dk, dv, dg (bf16) and dgamma_q,
    dgamma_k (fp32 [D]).  `grads` may supply preallocated outputs, `workspace` a uint8
    CUDA tensor of at least zgcm_attn_bwd_workspace_size(...) bytes.  `saved`: the store a
    zgcm_attn_fwd(saved=...) of the same inputs filled (zgcm_attn_bwd_saved).  `kernel_events`,
    a list of (begin, end) torch.cuda.Event pairs, brackets the backward's kernels in launch
    order (zgcm_attn_bwd_timed; names from zgcm_attn_bwd_kernel_names)."""
    import torch
    B, S, _, Hq, Hkv, D = _check_bwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, dout, grads, workspace, saved)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if grads is None:
        grads = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                     dg=torch.empty_like(g),
                     dgamma_q=torch.empty(D, dtype=torch.float32, device=q.device),
                     dgamma_k=torch.empty(D, dtype=torch.float32, device=q.device))
    need = zgcm_attn_bwd_workspace_size(B, S, Hq, Hkv, D, window)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
            _ptr(out), _ptr(lse), _ptr(dout), B, S, Hq, Hkv, D, int(rope_dims),
            float(rope_base), int(window), int(causal), float(eps), float(scale),
            _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["dg"]),
            _ptr(grads["dgamma_q"]), _ptr(grads["dgamma_k"]), _ptr(workspace),
            workspace.numel(), _stream(stream))
    arr, n_pairs = None, 0
    if kernel_events is not None:
        st_obj = stream if stream is not None else torch.cuda.current_stream()
        for pair in kernel_events:
            for e in pair:
                if not e.cuda_event:  # torch creates the CUDA event on its first record
                    e.record(st_obj)
        flat = [ctypes.c_void_p(e.cuda_event) for pair in kernel_events for e in pair]
        arr = (ctypes.c_void_p * max(1, len(flat)))(*flat)
        n_pairs = len(kernel_events)
    if saved is not None:
        st = load().zgcm_attn_bwd_saved(*args[:-1], _ptr(saved), saved.numel(), args[-1], arr, n_pairs)
        if st != ZGCM_OK:
            raise ZgcmError(st, "zgcm_attn_bwd_saved")
        return grads
    if kernel_events is None:
        st = load().zgcm_attn_bwd(*args)
    else:
        st = load().zgcm_attn_bwd_timed(*args, arr, n_pairs)
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_bwd")
    return grads


def zgcm_attn_fwd_rows(q, k, v, g, gamma_q, gamma_k, *, rope_dims=42, rope_base=10000.0, window,
                       causal=1, eps=1e-6, scale=None, out=None, lse=None, workspace=None, stream=None):
    """Forward of the query rows at the end of a longer key sequence: q, g [B,Sq,Hq,D] are
    positions S-Sq .. S-1 of k, v [B,S,Hkv,D] (S - Sq a multiple of 128 and window > 128 when
    Sq < S).  Returns (out bf16 [B,Sq,Hq,D], lse fp32 [B,Hq,Sq]), the rows of the whole
    sequence's forward."""
    import torch
    B, Sq, S, Hq, Hkv, D = _check_fwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, workspace, rows=True)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    need = zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D, rope_dims, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    st = load().zgcm_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
                                   B, Sq, S, Hq, Hkv, D, int(rope_dims), float(rope_base), int(window),
                                   int(causal), float(eps), float(scale), _ptr(out), _ptr(lse),
                                   ws_ptr, ws_bytes, _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_fwd_rows")
    return out, lse


def zgcm_attn_bwd_rows(q, k, v, g, gamma_q, gamma_k, out, lse, dout, *, rope_dims=42, rope_base=10000.0,
                       window, causal=1, eps=1e-6, scale=None, grads=None, workspace=None, stream=None):
    """Backward of zgcm_attn_fwd_rows: dq, dg of the query rows, dk, dv of every key row and
    dgamma_q, dgamma_k, each the part these query rows contribute (a dict as zgcm_attn_bwd)."""
    import torch
    B, Sq, S, Hq, Hkv, D = _check_bwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, dout, grads, workspace,
                                           rows=True)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if grads is None:
        grads = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                     dg=torch.empty_like(g),
                     dgamma_q=torch.empty(D, dtype=torch.float32, device=q.device),
                     dgamma_k=torch.empty(D, dtype=torch.float32, device=q.device))
    need = zgcm_attn_bwd_workspace_size(B, S, Hq, Hkv, D, window)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = load().zgcm_attn_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
                                   _ptr(out), _ptr(lse), _ptr(dout), B, Sq, S, Hq, Hkv, D, int(rope_dims),
                                   float(rope_base), int(window), int(causal), float(eps), float(scale),
                                   _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["dg"]),
                                   _ptr(grads["dgamma_q"]), _ptr(grads["dgamma_k"]), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_bwd_rows")
    return grads


def zgcm_attn_bwd_noalloc(q, k, v, g, gamma_q, gamma_k, out, lse, dout, *, rope_dims=42, rope_base=10000.0,
                          window=128, causal=1, eps=1e-6, scale=None, grads=None, stream=None):
    """zgcm_attn_bwd without a workspace: for callers that cannot allocate device memory,
    the library's fixed 64 MiB per-device scratch array is used instead (problems needing
    more raise ZgcmError with ZGCM_ERR_TOO_LARGE: at 32/8 heads and a window of at most 128,
    B*S <= 3117 tokens fit).  The call runs with q's device current, so the array used is
    that device's.  Calls that overlap on the GPU race."""
    import torch
    B, S, _, Hq, Hkv, D = _check_bwd_args(q, k, v, g, gamma_q, gamma_k, out, lse, dout, grads)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if grads is None:
        grads = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                     dg=torch.empty_like(g),
                     dgamma_q=torch.empty(D, dtype=torch.float32, device=q.device),
                     dgamma_k=torch.empty(D, dtype=torch.float32, device=q.device))
    with torch.cuda.device(q.device):
        st = load().zgcm_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma_q), _ptr(gamma_k),
                                          _ptr(out), _ptr(lse), _ptr(dout), B, S, Hq, Hkv, D, int(rope_dims),
                                          float(rope_base), int(window), int(causal), float(eps), float(scale),
                                          _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
                                          _ptr(grads["dg"]), _ptr(grads["dgamma_q"]), _ptr(grads["dgamma_k"]),
                                          _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_attn_bwd_noalloc")
    return grads


# ---------------------------------------------------------------- Muon optimiser (zgcm_muon.h)

# momentum, iterations, learning rate and weight decay of the ZGCM-1 summary, section
# "前置知识 / Muon 优化器"; the classical Newton–Schulz coefficients (the pages give none)
MUON_MOMENTUM, MUON_STEPS, MUON_LR, MUON_WEIGHT_DECAY = 0.9, 5, 2e-4, 0.1
MUON_COEFFS = (1.5, -0.5, 0.0)


def zgcm_muon_workspace_size(m, n) -> int:
    """Bytes of workspace zgcm_muon_step / zgcm_muon_orthogonalize need for an m x n matrix."""
    return int(load().zgcm_muon_workspace_size(int(m), int(n)))


def _muon_ws(m, n, workspace, device):
    import torch
    need = zgcm_muon_workspace_size(m, n)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    _check(workspace, "workspace", torch.uint8, 1, cuda=False)
    if not workspace.is_cuda or workspace.device != device:
        raise TypeError(f"workspace must be a CUDA tensor on the matrix's device ({device})")
    return workspace


def zgcm_muon_step(W, G, M, *, lr=MUON_LR, weight_decay=MUON_WEIGHT_DECAY, momentum=MUON_MOMENTUM,
                   steps=MUON_STEPS, coeffs=MUON_COEFFS, eps=1e-7, workspace=None, stream=None):
    """One Muon step in place: W fp32 [m, n], G bf16 [m, n], M fp32 [m, n] (momentum buffer)."""
    import torch
    _check(W, "W", torch.float32, 2, cuda=False)
    _need(G, "G", torch.bfloat16, W.shape)
    _need(M, "M", torch.float32, W.shape)
    _one_device(("W", W), ("G", G), ("M", M))
    m, n = W.shape
    ws = _muon_ws(m, n, workspace, W.device)
    a, b, c = (float(x) for x in coeffs)
    st = load().zgcm_muon_step(_ptr(W), _ptr(G), _ptr(M), m, n, float(lr), float(weight_decay), float(momentum),
                               int(steps), a, b, c, float(eps), _ptr(ws), ws.numel(), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_muon_step")
    return W, M


def zgcm_muon_orthogonalize(G, *, steps=MUON_STEPS, coeffs=MUON_COEFFS, eps=1e-7, out=None, workspace=None,
                            stream=None):
    """bf16 [m, n]: the Newton–Schulz iterate after `steps` steps from G / (||G||_F + eps)."""
    import torch
    _check(G, "G", torch.bfloat16, 2, cuda=False)
    if out is not None:
        _need(out, "out", torch.bfloat16, G.shape)
    _one_device(("G", G), ("out", out))
    m, n = G.shape
    if out is None:
        out = torch.empty_like(G)
    ws = _muon_ws(m, n, workspace, G.device)
    a, b, c = (float(x) for x in coeffs)
    st = load().zgcm_muon_orthogonalize(_ptr(G), _ptr(out), m, n, int(steps), a, b, c, float(eps), _ptr(ws),
                                        ws.numel(), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_muon_orthogonalize")
    return out


def zgcm_muon_gemm(A, B, *, D=None, alpha=1.0, beta=0.0, b_kn=False, out=None, stream=None):
    """C = alpha A op(B) + beta D in bf16 (fp32 accumulation): A [M, K]; B [K, N] if b_kn else
    [N, K] (C = A B^T)."""
    import torch
    _check(A, "A", torch.bfloat16, 2, cuda=False)
    _check(B, "B", torch.bfloat16, 2, cuda=False)
    M, K = A.shape
    N = B.shape[1] if b_kn else B.shape[0]
    if (B.shape[0] if b_kn else B.shape[1]) != K:
        raise TypeError("inner dimensions of A and B differ")
    if D is not None:
        _need(D, "D", torch.bfloat16, (M, N))
    if out is not None:
        _need(out, "out", torch.bfloat16, (M, N))
    _one_device(("A", A), ("B", B), ("D", D), ("out", out))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    st = load().zgcm_muon_gemm(_ptr(A), _ptr(B), _ptr(D), _ptr(out), M, N, K, float(alpha), float(beta),
                               1 if b_kn else 0, _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_muon_gemm")
    return out


# ---------------------------------------------------------------- projections (zgcm_proj.h)

def _proj_check(*named):
    """(name, tensor, shape) triples: contiguous bf16 of that shape (None: not given), then one
    CUDA device for all of them."""
    import torch
    for n, t, shape in named:
        if t is not None:
            _need(t, n, torch.bfloat16, shape)
    _one_device(*((n, t) for n, t, _ in named))


def zgcm_proj_qkvg_fwd(x, w_qkvg, *, Hq=32, Hkv=8, D=128, out=None, stream=None):
    """q, g [T, Hq*D] and k, v [T, Hkv*D] = the parts of x W_qkvg^T (x [T, d_model] bf16,
    W_qkvg [(2 Hq + 2 Hkv) D, d_model] bf16, the rows of W_q, W_k, W_v, W_g)."""
    import torch
    _check(x, "x", torch.bfloat16, 2, cuda=False)
    T, dm = x.shape
    widths = (Hq * D, Hkv * D, Hkv * D, Hq * D)
    if out is not None and len(out) != 4:
        raise TypeError("out must be the four tensors q, k, v, g")
    outs = (None,) * 4 if out is None else tuple(out)
    _proj_check(("x", x, (T, dm)), ("w_qkvg", w_qkvg, (sum(widths), dm)),
                *((n, t, (T, w)) for n, t, w in zip(("q", "k", "v", "g"), outs, widths)))
    if out is None:
        out = tuple(torch.empty((T, w), dtype=torch.bfloat16, device=x.device) for w in widths)
    st = load().zgcm_proj_qkvg_fwd(_ptr(x), _ptr(w_qkvg), T, dm, Hq, Hkv, D, *(_ptr(t) for t in out), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_proj_qkvg_fwd")
    return out


def zgcm_proj_qkvg_bwd(x, w_qkvg, dq, dk, dv, dg, *, Hq=32, Hkv=8, D=128, dx=None, dw=None, stream=None):
    """dx = [dq|dk|dv|dg] W_qkvg and dW_qkvg = [dq|dk|dv|dg]^T x (bf16)."""
    import torch
    _check(x, "x", torch.bfloat16, 2, cuda=False)
    T, dm = x.shape
    widths = (Hq * D, Hkv * D, Hkv * D, Hq * D)
    _proj_check(("x", x, (T, dm)), ("w_qkvg", w_qkvg, (sum(widths), dm)),
                *((n, t, (T, w)) for n, t, w in zip(("dq", "dk", "dv", "dg"), (dq, dk, dv, dg), widths)),
                ("dx", dx, (T, dm)), ("dw", dw, (sum(widths), dm)))
    dx = torch.empty_like(x) if dx is None else dx
    dw = torch.empty_like(w_qkvg) if dw is None else dw
    st = load().zgcm_proj_qkvg_bwd(_ptr(x), _ptr(w_qkvg), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), T, dm, Hq, Hkv,
                                   D, _ptr(dx), _ptr(dw), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_proj_qkvg_bwd")
    return dx, dw


def zgcm_proj_out_fwd(a, w_o, *, out=None, stream=None):
    """y [T, d_model] = a W_o^T (a [T, d_in], W_o [d_model, d_in], bf16)."""
    import torch
    _check(a, "a", torch.bfloat16, 2, cuda=False)
    _check(w_o, "w_o", torch.bfloat16, 2, cuda=False)
    T, din = a.shape
    dm = w_o.shape[0]
    _proj_check(("a", a, (T, din)), ("w_o", w_o, (dm, din)), ("out", out, (T, dm)))
    y = torch.empty((T, dm), dtype=torch.bfloat16, device=a.device) if out is None else out
    st = load().zgcm_proj_out_fwd(_ptr(a), _ptr(w_o), T, din, dm, _ptr(y), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_proj_out_fwd")
    return y


def zgcm_proj_out_bwd(a, w_o, dy, *, da=None, dw=None, stream=None):
    """da = dy W_o and dW_o = dy^T a (bf16)."""
    import torch
    _check(a, "a", torch.bfloat16, 2, cuda=False)
    _check(w_o, "w_o", torch.bfloat16, 2, cuda=False)
    T, din = a.shape
    dm = w_o.shape[0]
    _proj_check(("a", a, (T, din)), ("w_o", w_o, (dm, din)), ("dy", dy, (T, dm)), ("da", da, (T, din)),
                ("dw", dw, (dm, din)))
    da = torch.empty_like(a) if da is None else da
    dw = torch.empty_like(w_o) if dw is None else dw
    st = load().zgcm_proj_out_bwd(_ptr(a), _ptr(w_o), _ptr(dy), T, din, dm, _ptr(da), _ptr(dw), _stream(stream))
    if st != ZGCM_OK:
        raise ZgcmError(st, "zgcm_proj_out_bwd")
    return da, dw
