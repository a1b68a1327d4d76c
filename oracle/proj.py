"""fp64 CPU oracle of the projections around the gated attention layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this module; it shares no code with the GPU library.  Each function is the definition written
out with one library matmul per product, in float64.

q, k, v and the gate logits g are linear maps of the layer input x (ZGCM-1 summary, section
"核心方法": hidden size 4096, 32 query and 8 KV heads of 128; the source of g is not stated, and
the plainest reading is a linear map of x like the others); the attention output goes through
an output projection.  No biases.  W_qkvg stacks the rows of W_q, W_k, W_v, W_g.  Pinned by
``tests/test_oracle_proj.py`` (torch autograd of a Linear layer, the split order by hand).
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to(torch.float64).cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def qkvg_forward(x, w_qkvg, wq: int, wkv: int):
    """q, k, v, g = the column blocks of x W_qkvg^T of widths wq, wkv, wkv, wq."""
    y = _f64(x) @ _f64(w_qkvg).T
    return y[:, :wq], y[:, wq:wq + wkv], y[:, wq + wkv:wq + 2 * wkv], y[:, wq + 2 * wkv:]


def qkvg_backward(x, w_qkvg, dq, dk, dv, dg):
    """dx = [dq|dk|dv|dg] W_qkvg and dW_qkvg = [dq|dk|dv|dg]^T x."""
    dy = np.concatenate([_f64(t) for t in (dq, dk, dv, dg)], axis=1)
    return dy @ _f64(w_qkvg), dy.T @ _f64(x)


def out_forward(a, w_o):
    """y = a W_o^T."""
    return _f64(a) @ _f64(w_o).T


def out_backward(a, w_o, dy):
    """da = dy W_o and dW_o = dy^T a."""
    dy = _f64(dy)
    return dy @ _f64(w_o), dy.T @ _f64(a)


def proj_flops(T: int, d_model: int, wq: int, wkv: int, d_in: int) -> dict:
    """Multiply-add FLOPs (2 per multiply-add) of each call."""
    n = 2 * (wq + wkv)
    return {"qkvg_fwd": 2 * T * d_model * n, "qkvg_bwd": 4 * T * d_model * n,
            "out_fwd": 2 * T * d_in * d_model, "out_bwd": 4 * T * d_in * d_model}
