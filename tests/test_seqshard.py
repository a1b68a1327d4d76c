"""Sequence sharding of the layer (global_attention_b200.seqshard) as gloo process groups on
the CPU: each rank computes its rows with the fp64 oracle through the halo exchange (sliding
windows) or the gathered earlier rows (any window, the global layer among them), and the
results must equal the unsharded oracle on the whole sequence."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops(calls=None):
    """The layer's entry points restated with the fp64 oracle: fwd, bwd and the query-row pair
    (query rows at the end of the key rows: zero query rows in front, results sliced), each
    call counted in `calls` by name."""
    import oracle

    def count(name):
        if calls is not None:
            calls[name] = calls.get(name, 0) + 1

    def fwd(q, k, v, g, gq, gk, *, window, **kw):
        count("fwd")
        out, lse = oracle.Problem(q, k, v, g, gq, gk, window=window, **kw).forward()
        return torch.from_numpy(out), torch.from_numpy(lse)

    def bwd(q, k, v, g, gq, gk, out, lse, dout, *, window, **kw):
        count("bwd")
        r = oracle.Problem(q, k, v, g, gq, gk, window=window, **kw).backward(dout)
        return {n: torch.from_numpy(x) for n, x in r.items()}

    def pad(x, h):
        return torch.cat([torch.zeros((x.shape[0], h) + tuple(x.shape[2:]), dtype=x.dtype), x], 1)

    def fwd_rows(q, k, v, g, gq, gk, *, window, **kw):
        count("fwd_rows")
        h = k.shape[1] - q.shape[1]
        out, lse = oracle.Problem(pad(q, h), k, v, pad(g, h), gq, gk, window=window, **kw).forward()
        return torch.from_numpy(out[:, h:]), torch.from_numpy(lse[:, :, h:])

    def bwd_rows(q, k, v, g, gq, gk, out, lse, dout, *, window, **kw):
        count("bwd_rows")
        h = k.shape[1] - q.shape[1]
        r = oracle.Problem(pad(q, h), k, v, pad(g, h), gq, gk, window=window, **kw).backward(pad(dout, h))
        r = {n: torch.from_numpy(x) for n, x in r.items()}
        for n in ("dq", "dg"):
            r[n] = r[n][:, h:]
        return r

    return fwd, bwd, fwd_rows, bwd_rows


def _rank_main(rank, world, port, L, W, results, mode="halo", calls_out=None):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from datetime import timedelta
    import oracle
    from global_attention_b200 import seqshard
    from global_attention_b200.synth import make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        kw = dict(rope_dims=8, rope_base=10000.0)
        B, Hq, Hkv, D = 2, 4, 2, 16
        t = make_inputs(B, world * L, Hq=Hq, Hkv=Hkv, D=D, seed=21, with_dout=True)
        rows = slice(rank * L, (rank + 1) * L)
        mine = {n: t[n][:, rows].contiguous() for n in ("q", "k", "v", "g", "dout")}
        calls = {}
        ops = _oracle_ops(calls)
        fwd = seqshard.halo_forward if mode == "halo" else seqshard.gathered_forward
        bwd = seqshard.halo_backward if mode == "halo" else seqshard.gathered_backward
        out, lse, ctx = fwd(mine["q"], mine["k"], mine["v"], mine["g"], t["gamma_q"], t["gamma_k"], window=W,
                            ops=ops, **kw)
        gr = bwd(ctx, mine["dout"], t["gamma_q"], t["gamma_k"], ops=ops)
        # the whole sequence at once
        P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], window=W, **kw)
        ref_out, ref_lse = P.forward()
        ref = P.backward(t["dout"])
        err = {
            "out": np.abs(out.numpy() - ref_out[:, rows]).max(),
            "lse": np.abs(lse.numpy() - ref_lse[:, :, rows]).max(),
        }
        for n in ("dq", "dk", "dv", "dg"):
            err[n] = np.abs(gr[n].numpy() - ref[n][:, rows]).max()
        for n in ("dgamma_q", "dgamma_k"):
            err[n] = np.abs(gr[n].numpy() - ref[n]).max() / max(1.0, np.abs(ref[n]).max())
        results[rank] = {k: float(v) for k, v in err.items()}
        if calls_out is not None:
            calls_out[rank] = dict(calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,W", [(2, 24, 16), (3, 20, 16), (3, 15, 16), (2, 9, 1)])
def test_halo_sharding_equals_whole_sequence(world, L, W):
    """Ranks 0..world-1 each hold L rows; window W reaches W - 1 rows into the previous rank
    (L = W - 1: exactly one whole rank of halo; W = 1: no halo, only the d_gamma sum).  Every
    output and gradient equals the unsharded oracle to fp64 rounding (RoPE at shifted
    positions differs only in the rounding of its angles)."""
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), L, W, results), nprocs=world, join=True)
    assert len(results) == world
    for rank in range(world):
        for name, e in results[rank].items():
            assert e < 1e-9, (rank, name, e)


@pytest.mark.parametrize("world,L,W", [(2, 16, 10**6), (3, 12, 36), (3, 10, 16), (3, 12, 8), (2, 9, 1)])
def test_gathered_sharding_equals_whole_sequence(world, L, W):
    """Windows that reach past the previous rank: the global layer (W >= the whole sequence),
    W - 1 >= 2 L (every earlier row), and L = 10, W = 16, where rank 2's window covers rank 1
    and rows 5..9 of rank 0; a short window and W = 1 take the same path.  Every output and
    gradient equals the unsharded oracle to fp64 rounding."""
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), L, W, results, "gathered"), nprocs=world, join=True)
    assert len(results) == world
    for rank in range(world):
        for name, e in results[rank].items():
            assert e < 1e-9, (rank, name, e)


@pytest.mark.parametrize("world,L,W", [(2, 128, 10**6), (3, 128, 200)])
def test_gathered_sharding_query_rows(world, L, W):
    """With a window wider than 128 and rank boundaries on 128 rows the gathered shards go
    through the query-row entry points (this rank's rows as the last ones of the gathered key
    rows, whose start is rounded down to a 128-row boundary; no zero query rows): every rank
    after the first calls them, and every output and gradient still equals the unsharded
    oracle (global layer; W = 200, where rank 2's start 57 becomes 0 and rank 1's 0 stays)."""
    mgr = mp.get_context("spawn").Manager()
    results, calls = mgr.dict(), mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), L, W, results, "gathered", calls), nprocs=world, join=True)
    assert len(results) == world
    for rank in range(world):
        for name, e in results[rank].items():
            assert e < 1e-9, (rank, name, e)
        if rank > 0:
            assert calls[rank] == {"fwd_rows": 1, "bwd_rows": 1}, calls[rank]
        else:
            assert calls[rank] == {"fwd": 1, "bwd": 1}, calls[rank]


def test_halo_needs_window_rows_per_rank():
    """A rank with fewer than W - 1 rows would need rows of two ranks back: refused."""
    sys.path.insert(0, ROOT)
    from global_attention_b200 import seqshard

    # a two-rank group seen from rank 1, without a process group
    orig = dist.get_rank, dist.get_world_size
    try:
        dist.get_rank = lambda group=None: 1
        dist.get_world_size = lambda group=None: 2
        x = torch.zeros(1, 10, 4, 16, dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            seqshard.halo_forward(x, x[:, :, :2], x[:, :, :2], x, torch.ones(16), torch.ones(16), window=16,
                                  ops=(None, None))
    finally:
        dist.get_rank, dist.get_world_size = orig
