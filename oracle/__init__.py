"""fp64 CPU oracle of the ZGCM-1 gated window-attention layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  It shares no code with the GPU library: the arithmetic lives in
``zgcm_oracle.c`` (plain double-precision definitions) and this module only converts
arrays and calls it through ctypes.

Parity status: every function here is pinned by ``tests/test_oracle.py`` (brute force on
tiny inputs, closed forms, invariants, finite differences, torch autograd and a torch
SDPA special case), except two readings the pages cannot decide — the RoPE pairing
convention and the gate formula — which are "parity unpinned" against the real model.

Page citations for what is computed are in ``zgcm_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zgcm_oracle.c")
_LIB = os.path.join(_HERE, "libzgcm_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, OpenMP, strict IEEE double; no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("gamma_q", ctypes.c_void_p), ("gamma_k", ctypes.c_void_p),
                ("B", ctypes.c_int64), ("S", ctypes.c_int64), ("Hq", ctypes.c_int64),
                ("Hkv", ctypes.c_int64), ("D", ctypes.c_int64), ("R", ctypes.c_int64),
                ("W", ctypes.c_int64), ("base", ctypes.c_double), ("eps", ctypes.c_double),
                ("scale", ctypes.c_double)]


def _bind(lib):
    P = ctypes.POINTER(_Problem)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.zo_forward.argtypes = [P, vp, i64, vp, vp]
    lib.zo_backward_qrows.argtypes = [P, vp, vp, i64, vp, vp]
    lib.zo_backward_krows.argtypes = [P, vp, vp, i64, vp, vp]
    lib.zo_backward_full.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.zo_prologue_row.argtypes = [P, vp, vp, i64, vp]
    lib.zo_prologue_row.restype = None
    lib.zo_num_threads.argtypes = []
    for f in (lib.zo_forward, lib.zo_backward_qrows, lib.zo_backward_krows, lib.zo_backward_full,
              lib.zo_num_threads):
        f.restype = ctypes.c_int
    return lib


class using_library:
    """Temporarily route every oracle call to another build of zgcm_oracle.c (the pin tests
    use it to check that planted mistakes are caught)."""

    def __init__(self, path: str):
        self.lib = _bind(ctypes.CDLL(path))

    def __enter__(self):
        global _lib
        self.saved, _lib = _lib, self.lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def num_threads() -> int:
    return int(_load().zo_num_threads())


def _f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (bf16/fp32/fp64) or array to contiguous float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().to(dtype=__import__("torch").float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Problem:
    """Inputs of one layer call, upcast once to float64 and kept alive for the C side."""

    def __init__(self, q, k, v, g, gamma_q, gamma_k, *, rope_dims=42, rope_base=10000.0,
                 window=128, eps=1e-6, scale=None):
        self.q, self.k, self.v, self.g = _f64(q), _f64(k), _f64(v), _f64(g)
        self.gamma_q, self.gamma_k = _f64(gamma_q), _f64(gamma_k)
        B, S, Hq, D = self.q.shape
        Hkv = self.k.shape[2]
        assert self.k.shape == (B, S, Hkv, D) and self.v.shape == self.k.shape
        assert self.g.shape == self.q.shape
        self.shape = (B, S, Hq, Hkv, D)
        if scale is None:
            scale = 1.0 / np.sqrt(D)
        self.c = _Problem(_ptr(self.q).value, _ptr(self.k).value, _ptr(self.v).value,
                          _ptr(self.g).value, _ptr(self.gamma_q).value, _ptr(self.gamma_k).value,
                          B, S, Hq, Hkv, D, int(rope_dims), int(window), float(rope_base),
                          float(eps), float(scale))

    def set_window(self, window: int):
        """Reuse the upcast inputs for another window size."""
        self.c.W = int(window)

    def _rows(self, rows):
        if rows is None:
            return None, self.shape[0] * self.shape[1]
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        return r, len(r)

    def forward(self, rows=None):
        """out, lse.  rows=None: out [B,S,Hq,D], lse [B,Hq,S].
        rows = flat indices b*S+i: out [n,Hq,D], lse [n,Hq]."""
        B, S, Hq, Hkv, D = self.shape
        r, n = self._rows(rows)
        out = np.zeros((n, Hq, D))
        lse = np.zeros((n, Hq))
        rc = _load().zo_forward(ctypes.byref(self.c), None if r is None else _ptr(r), n,
                                _ptr(out), _ptr(lse))
        if rc:
            raise RuntimeError(f"oracle forward failed ({rc})")
        if rows is None:
            return out.reshape(B, S, Hq, D), lse.reshape(B, S, Hq).transpose(0, 2, 1).copy()
        return out, lse

    def backward_qrows(self, dout, rows=None):
        """dq, dg for the listed query rows (shapes as in forward)."""
        B, S, Hq, Hkv, D = self.shape
        do = _f64(dout)
        r, n = self._rows(rows)
        dq = np.zeros((n, Hq, D))
        dg = np.zeros((n, Hq, D))
        rc = _load().zo_backward_qrows(ctypes.byref(self.c), _ptr(do), None if r is None else _ptr(r),
                                       n, _ptr(dq), _ptr(dg))
        if rc:
            raise RuntimeError(f"oracle backward_qrows failed ({rc})")
        if rows is None:
            return dq.reshape(B, S, Hq, D), dg.reshape(B, S, Hq, D)
        return dq, dg

    def backward_krows(self, dout, rows=None):
        """dk, dv for the listed key rows: [n,Hkv,D] (or [B,S,Hkv,D] when rows=None)."""
        B, S, Hq, Hkv, D = self.shape
        do = _f64(dout)
        r, n = self._rows(rows)
        dk = np.zeros((n, Hkv, D))
        dv = np.zeros((n, Hkv, D))
        rc = _load().zo_backward_krows(ctypes.byref(self.c), _ptr(do), None if r is None else _ptr(r),
                                       n, _ptr(dk), _ptr(dv))
        if rc:
            raise RuntimeError(f"oracle backward_krows failed ({rc})")
        if rows is None:
            return dk.reshape(B, S, Hkv, D), dv.reshape(B, S, Hkv, D)
        return dk, dv

    def backward(self, dout):
        """Full backward: dict of dq, dk, dv, dg, dgamma_q, dgamma_k."""
        B, S, Hq, Hkv, D = self.shape
        do = _f64(dout)
        dq = np.zeros((B, S, Hq, D)); dg = np.zeros((B, S, Hq, D))
        dk = np.zeros((B, S, Hkv, D)); dv = np.zeros((B, S, Hkv, D))
        dgq = np.zeros(D); dgk = np.zeros(D)
        rc = _load().zo_backward_full(ctypes.byref(self.c), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                                      _ptr(dg), _ptr(dgq), _ptr(dgk))
        if rc:
            raise RuntimeError(f"oracle backward failed ({rc})")
        return dict(dq=dq, dk=dk, dv=dv, dg=dg, dgamma_q=dgq, dgamma_k=dgk)

    def prologue_row(self, x, gamma, pos):
        """RoPE(gamma * x / rms(x)) of one row at position pos."""
        x = _f64(x); gm = _f64(gamma)
        y = np.zeros_like(x)
        _load().zo_prologue_row(ctypes.byref(self.c), _ptr(x), _ptr(gm), int(pos), _ptr(y))
        return y


def forward(q, k, v, g, gamma_q, gamma_k, rows=None, **kw):
    return Problem(q, k, v, g, gamma_q, gamma_k, **kw).forward(rows)


def kv_cache_bytes_per_token(n_growing_layers: int, n_kv_heads: int = 8, head_dim: int = 128,
                             bytes_per_elem: int = 2) -> int:
    """KV-cache bytes one more token adds: K and V of every layer whose cache grows with
    the context.  Full attention: all 32 layers grow; the 5:1 hybrid: only the 5 global
    layers grow, the 27 window layers keep a fixed 128-token cache (shibing624 review,
    section "架构": 128 KiB vs 20 KiB per token, 32 GiB vs 5 GiB at 256K)."""
    return n_growing_layers * n_kv_heads * head_dim * 2 * bytes_per_elem
