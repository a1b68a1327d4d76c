"""Planted mistakes: each mutant of the oracle source (a dropped term, a wrong sign or
index, a wrong constant) is compiled on the CPU and must fail at least one of the checks
the pins use — brute force, finite differences / autograd, closed forms."""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from global_attention_b200.synth import make_inputs
from tests.brute import brute_forward, torch_naive_forward

SRC = os.path.join(os.path.dirname(oracle.__file__), "zgcm_oracle.c")

MUTANTS = {
    "rmsnorm drops eps": ("sqrt(ss / (double)D + P->eps)", "sqrt(ss / (double)D)"),
    "rope sign": ("y[t] = y1 * c - y2 * s;", "y[t] = y1 * c + y2 * s;"),
    "rope theta denominator": ("-2.0 * (double)t / (double)P->R", "-2.0 * (double)t / (double)P->D"),
    "window off by one": ("int64_t lo = i - P->W + 1;", "int64_t lo = i - P->W;"),
    "gqa map": ("return h / (P->Hq / P->Hkv);", "return h % P->Hkv;"),
    "gate dropped": ("o[d] = sigmoid(gr[d]) * A[d];", "o[d] = A[d];"),
    "lse drops log-sum": ("*lse = m + log(l);", "*lse = m;"),
    "dg drops (1 - sigmoid)": ("dout_row[d] * A[d] * sg * (1.0 - sg)", "dout_row[d] * A[d] * sg"),
    "dS drops Delta": ("ds[t] = p[t] * (ds[t] - delta);", "ds[t] = p[t] * ds[t];"),
    "rmsnorm bwd drops mean term": ("dx[d] = (dy[d] * gamma[d] - xhat[d] * m) / r;", "dx[d] = (dy[d] * gamma[d]) / r;"),
    "rope bwd transpose sign": ("dy[t] = d1 * c + d2 * s;", "dy[t] = d1 * c - d2 * s;"),
    "dk drops scale": ("dkh[j * D + d] += P->scale * dsj * qh[d];", "dkh[j * D + d] += dsj * qh[d];"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old}"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(path_c), "-lm"],
                   check=True)
    return str(so)


def _checks_pass():
    """The pin checks in miniature; returns True if every one passes."""
    S, W, Hq, Hkv, D, R = 21, 5, 4, 2, 8, 4
    t = make_inputs(1, S, Hq=Hq, Hkv=Hkv, D=D, seed=7, with_dout=True)
    f = lambda x: x.to(torch.float64).numpy()
    kw = dict(rope_dims=R, rope_base=100.0, window=W, eps=1e-2)
    P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], **kw)
    out, lse = P.forward()
    bout, blse = brute_forward(f(t["q"]), f(t["k"]), f(t["v"]), f(t["g"]), f(t["gamma_q"]), f(t["gamma_k"]),
                               R=R, base=100.0, W=W, eps=1e-2)
    if not (np.allclose(out, bout, atol=1e-12, rtol=0) and np.allclose(lse, blse, atol=1e-12, rtol=0)):
        return False
    leaves = {n: t[n].double().clone().requires_grad_(True) for n in ("q", "k", "v", "g", "gamma_q", "gamma_k")}
    o = torch_naive_forward(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["gamma_q"],
                            leaves["gamma_k"], R, 100.0, W, 1e-2, 1.0 / math.sqrt(D))
    (o * t["dout"].double()).sum().backward()
    full = P.backward(t["dout"])
    for ours, theirs in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"), ("dgamma_q", "gamma_q"),
                         ("dgamma_k", "gamma_k")):
        if not np.allclose(full[ours], leaves[theirs].grad.numpy(), rtol=1e-9, atol=1e-10):
            return False
    return True


def test_unmutated_oracle_passes_the_checks():
    assert _checks_pass()


def _run_checks_with(so: str) -> int:
    """Run the checks against library `so` in a fresh process (a mutant may write out of
    bounds of its own buffers); returns 0 when every check passes."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; sys.path.insert(0, %r); import oracle; "
            "from tests.test_oracle_mutants import _checks_pass; "
            "ctx = oracle.using_library(%r); ctx.__enter__(); "
            "sys.exit(0 if _checks_pass() else 3)") % (root, so)
    return subprocess.run([sys.executable, "-c", code], capture_output=True).returncode


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    rc = _run_checks_with(so)
    assert rc != 0, f"mutant '{name}' passed every check"
