"""Tolerances and helpers for GPU-vs-oracle parity (shared by the -m gpu tests).

Tolerance (stated by the layer's target, and derived where it states none):
  bf16 outputs and gradients (out, dq, dk, dv, dg): max-abs <= 2e-2 AND
      rel-RMS = ||x - ref||_2 / ||ref||_2 <= 5e-3.
  lse (fp32): max-abs <= 2e-2 (own choice: lse is a log-sum, its error is the relative
      error of the row sum, which the bf16 rounding of q_hat, k_hat bounds near 1e-2).
  d_gamma (fp32, a sum over up to 2M rows, magnitude 1e1-1e2): rel-RMS <= 5e-3 and
      max-abs <= 2e-2 * max|ref| (an absolute 2e-2 is meaningless at that scale).
  A reference that is identically zero in exact arithmetic (dq when every query sees a
  single key: one-token sequences, window 1, and with it d_gamma_q) has an RMS at fp64
  rounding level; a relative measure against it is undefined, so when the reference RMS is
  below ZERO_RMS the relative bound is dropped and max-abs is checked against the absolute
  bf16 bound 2e-2 (for d_gamma too: 2e-2 * max|ref| would be a bound at fp64 rounding level).
"""
import numpy as np
import torch

BF16_ATOL = 2e-2
BF16_RRMS = 5e-3
LSE_ATOL = 2e-2
ZERO_RMS = 1e-9


def f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def errors(got, ref):
    got, ref = f64(got), f64(ref)
    diff = got - ref
    maxabs = float(np.abs(diff).max()) if diff.size else 0.0
    nref = float(np.linalg.norm(ref))
    rrms = float(np.linalg.norm(diff) / nref) if nref > 0 else float(np.linalg.norm(diff))
    return maxabs, rrms


def assert_bf16_close(name, got, ref, atol=BF16_ATOL, rrms=BF16_RRMS):
    g = f64(got)
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    m, r = errors(g, ref)
    ref = f64(ref)
    if ref.size and float(np.sqrt(np.mean(ref * ref))) < ZERO_RMS:
        r = 0.0  # exactly-zero reference: max-abs only
    assert m <= atol and r <= rrms, f"{name}: max-abs {m:.3e} (<= {atol}), rel-RMS {r:.3e} (<= {rrms})"
    return m, r


def assert_lse_close(name, got, ref, atol=LSE_ATOL):
    m, _ = errors(got, ref)
    assert m <= atol, f"{name}: max-abs {m:.3e} (<= {atol})"
    return m


def assert_dgamma_close(name, got, ref):
    ref = f64(ref)
    m, r = errors(got, ref)
    lim = 2e-2 * float(np.abs(ref).max())
    if float(np.sqrt(np.mean(ref * ref))) < ZERO_RMS:
        r, lim = 0.0, BF16_ATOL  # exactly-zero reference (dq == 0 everywhere): absolute bound only
    assert m <= lim and r <= BF16_RRMS, f"{name}: max-abs {m:.3e} (<= {lim:.3e}), rel-RMS {r:.3e}"
    return m, r
