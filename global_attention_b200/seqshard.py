"""Sequence-sharded layer: one long sequence split over the ranks of a process group, rank r
holding positions [r L, (r + 1) L) of every batch row.

A sliding window of W keys reaches W - 1 rows back, so each rank needs only the last W - 1
key and value rows of the rank before it (a halo).  The forward receives that halo and runs
the layer on [halo; own rows] with zero query and gate rows under the halo, whose outputs are
dropped; the backward runs on the same extended rows with zero output gradient there, sends
the halo's dk and dv back to the rank that owns those rows (which adds them to its own), and
sums d_gamma over the ranks.  Two facts make this exact:

* attention scores depend on positions only through their differences (RoPE rotates both
  rows by their own position, and a rotation by a then b has the dot product of a rotation by
  a - b), so the extended rows may be numbered from 0 on every rank;
* the gradients of a key row, and each row's share of d_gamma, are sums over the query rows
  that see it, so the parts computed on two ranks add.

Zero query rows take no part in any other row's result, and with zero output gradient they
contribute nothing to any gradient.  The exchange is one send and one receive of
2 (W - 1) B Hkv D values per rank and direction (torch.distributed point-to-point: NCCL over
NVLink on GPUs, gloo on the CPU); there is no collective on the data path except the sum of
d_gamma (2 x D values).

A window longer than a rank's rows (the global layer, W >= S, among them) reaches further
back: gathered_forward / gathered_backward gather every rank's key and value rows, run the
layer on the rows the window reaches ([start, (r + 1) L), start = max(0, r L - (W - 1)),
numbered from 0) for this rank's query rows, and return the earlier rows' key gradients to
their owners through one sum over the ranks.  With a window wider than 128 and r L a
multiple of 128, start is rounded down to a multiple of 128 and the query-row entry points
(zgcm_attn_fwd_rows / zgcm_attn_bwd_rows) take this rank's rows as the last ones of the
gathered sequence, so no query row before them is computed; otherwise zero query rows stand
before this rank's and their results are dropped.

The compute is a tuple of callables with the signatures of zgcm_attn_fwd, zgcm_attn_bwd and
(optionally) zgcm_attn_fwd_rows, zgcm_attn_bwd_rows of this package (the default); the tests
pass others to check the sharding on the CPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _default_ops():
    import global_attention_b200 as ga
    return ga.zgcm_attn_fwd, ga.zgcm_attn_bwd, ga.zgcm_attn_fwd_rows, ga.zgcm_attn_bwd_rows


def _ops4(ops):
    """(fwd, bwd, fwd_rows or None, bwd_rows or None)."""
    ops = tuple(ops or _default_ops())
    return ops + (None,) * (4 - len(ops))


def _exchange(send, recv_shape, like, to_rank, from_rank, group):
    """Send `send` to `to_rank` (None: nothing) and receive a tensor of `recv_shape` from
    `from_rank` (None: nothing), concurrently.  Returns the received tensor or None."""
    reqs, got = [], None
    if to_rank is not None:
        reqs.append(dist.isend(send.contiguous(), dst=dist.get_global_rank(group, to_rank)
                               if group is not None else to_rank, group=group))
    if from_rank is not None:
        got = torch.empty(recv_shape, dtype=like.dtype, device=like.device)
        reqs.append(dist.irecv(got, src=dist.get_global_rank(group, from_rank)
                               if group is not None else from_rank, group=group))
    for r in reqs:
        r.wait()
    return got


class HaloContext:
    """What the backward of one sharded forward needs."""

    def __init__(self, h, ext, out_ext, lse_ext, window, kw):
        self.h, self.ext, self.out_ext, self.lse_ext, self.window, self.kw = h, ext, out_ext, lse_ext, window, kw


def halo_forward(q, k, v, g, gamma_q, gamma_k, *, window, group=None, ops=None, **kw):
    """Forward of this rank's rows.  q, g [B, L, Hq, D]; k, v [B, L, Hkv, D] are the rows of
    positions r L .. r L + L - 1; every rank has the same L >= window - 1.  Returns out
    [B, L, Hq, D], lse [B, Hq, L] of those rows and a HaloContext for halo_backward."""
    fwd = _ops4(ops)[0]
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, L = q.shape[0], q.shape[1]
    h = window - 1
    if world > 1 and L < h:
        raise ValueError(f"each rank needs at least window - 1 = {h} rows (has {L})")
    tail = torch.stack([k[:, L - h:], v[:, L - h:]]) if world > 1 and h > 0 else None
    halo = None
    if world > 1 and h > 0:
        halo = _exchange(tail, (2,) + tuple(k[:, :h].shape), k,
                         rank + 1 if rank + 1 < world else None, rank - 1 if rank > 0 else None, group)
    if halo is None:  # first rank (or no halo): the rows alone
        out, lse = fwd(q, k, v, g, gamma_q, gamma_k, window=window, **kw)
        return out, lse, HaloContext(0, (q, k, v, g), out, lse, window, kw)
    zq = torch.zeros((B, h) + tuple(q.shape[2:]), dtype=q.dtype, device=q.device)
    ext = (torch.cat([zq, q], 1).contiguous(), torch.cat([halo[0], k], 1).contiguous(),
           torch.cat([halo[1], v], 1).contiguous(), torch.cat([zq, g], 1).contiguous())
    out_ext, lse_ext = fwd(*ext, gamma_q, gamma_k, window=window, **kw)
    return (out_ext[:, h:].contiguous(), lse_ext[:, :, h:].contiguous(),
            HaloContext(h, ext, out_ext, lse_ext, window, kw))


def halo_backward(ctx, dout, gamma_q, gamma_k, *, group=None, ops=None):
    """Backward of halo_forward on this rank: dict of dq, dk, dv, dg for its rows and
    dgamma_q, dgamma_k of the whole sequence (summed over the ranks)."""
    bwd = _ops4(ops)[1]
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    h = ctx.h
    q, k, v, g = ctx.ext
    if h > 0:
        zd = torch.zeros((dout.shape[0], h) + tuple(dout.shape[2:]), dtype=dout.dtype, device=dout.device)
        dout = torch.cat([zd, dout], 1).contiguous()
    gr = bwd(q, k, v, g, gamma_q, gamma_k, ctx.out_ext, ctx.lse_ext, dout, window=ctx.window, **ctx.kw)
    res = {n: gr[n][:, h:].contiguous() for n in ("dq", "dk", "dv", "dg")}
    if world > 1 and ctx.window > 1:
        hw = ctx.window - 1
        # the halo's key gradients go back to the rank that owns those rows
        back = torch.stack([gr["dk"][:, :h], gr["dv"][:, :h]]) if h > 0 else None
        L = res["dk"].shape[1]
        got = _exchange(back, (2,) + tuple(res["dk"][:, L - hw:].shape), res["dk"],
                        rank - 1 if rank > 0 else None, rank + 1 if rank + 1 < world else None, group)
        if got is not None:
            for i, n in enumerate(("dk", "dv")):
                tail = res[n][:, L - hw:]
                acc = torch.float64 if tail.dtype == torch.float64 else torch.float32
                res[n][:, L - hw:] = (tail.to(acc) + got[i].to(acc)).to(tail.dtype)
    dgam = torch.stack([gr["dgamma_q"], gr["dgamma_k"]]).contiguous()
    if world > 1:
        dist.all_reduce(dgam, group=group)
    res["dgamma_q"], res["dgamma_k"] = dgam[0], dgam[1]
    return res


def gathered_forward(q, k, v, g, gamma_q, gamma_k, *, window, group=None, ops=None, **kw):
    """Forward of this rank's rows for any window: the key and value rows of the earlier
    ranks that the window reaches are gathered (all ranks' rows travel; each keeps what it
    needs).  Shapes as halo_forward; every rank has the same L."""
    fwd, _, fwd_rows, _ = _ops4(ops)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, L = q.shape[0], q.shape[1]
    start = max(0, rank * L - (window - 1))
    # the query-row kernels take a first query row on a 128-row boundary, windows wider than 128
    rows = fwd_rows is not None and window > 128 and (rank * L) % 128 == 0
    if rows:
        start -= start % 128
    h = rank * L - start
    if world == 1 or h == 0:
        out, lse = fwd(q, k, v, g, gamma_q, gamma_k, window=window, **kw)
        kv_all = None
        if world > 1:  # the others still gather: take part with this rank's rows
            kv_all = [torch.empty_like(torch.stack([k, v])) for _ in range(world)]
            dist.all_gather(kv_all, torch.stack([k, v]).contiguous(), group=group)
        return out, lse, HaloContext(0, (q, k, v, g), out, lse, window, dict(kw, _start=start))
    kv_all = [torch.empty_like(torch.stack([k, v])) for _ in range(world)]
    dist.all_gather(kv_all, torch.stack([k, v]).contiguous(), group=group)
    before = torch.cat(kv_all[:rank], 2)[:, :, start:]  # [2, B, h, Hkv, D]
    if rows:
        ext_k = torch.cat([before[0], k], 1).contiguous()
        ext_v = torch.cat([before[1], v], 1).contiguous()
        out, lse = fwd_rows(q, ext_k, ext_v, g, gamma_q, gamma_k, window=window, **kw)
        return out, lse, HaloContext(h, (q, ext_k, ext_v, g), out, lse, window, dict(kw, _start=start, _rows=True))
    zq = torch.zeros((B, h) + tuple(q.shape[2:]), dtype=q.dtype, device=q.device)
    ext = (torch.cat([zq, q], 1).contiguous(), torch.cat([before[0], k], 1).contiguous(),
           torch.cat([before[1], v], 1).contiguous(), torch.cat([zq, g], 1).contiguous())
    out_ext, lse_ext = fwd(*ext, gamma_q, gamma_k, window=window, **kw)
    return (out_ext[:, h:].contiguous(), lse_ext[:, :, h:].contiguous(),
            HaloContext(h, ext, out_ext, lse_ext, window, dict(kw, _start=start)))


def gathered_backward(ctx, dout, gamma_q, gamma_k, *, group=None, ops=None):
    """Backward of gathered_forward: this rank's dq, dk, dv, dg and the whole sequence's
    dgamma_q, dgamma_k.  The key and value gradients of all rows are summed over the ranks
    (each rank contributes the rows its window reached) and each keeps its own."""
    _, bwd, _, bwd_rows = _ops4(ops)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    kw = dict(ctx.kw)
    start = kw.pop("_start")
    rows = kw.pop("_rows", False)
    h = ctx.h
    q, k, v, g = ctx.ext
    if rows:  # this rank's query rows only, the gathered key rows before them
        gr = bwd_rows(q, k, v, g, gamma_q, gamma_k, ctx.out_ext, ctx.lse_ext, dout, window=ctx.window, **kw)
        res = {n: gr[n].contiguous() for n in ("dq", "dg")}
    else:
        if h > 0:
            zd = torch.zeros((dout.shape[0], h) + tuple(dout.shape[2:]), dtype=dout.dtype, device=dout.device)
            dout = torch.cat([zd, dout], 1).contiguous()
        gr = bwd(q, k, v, g, gamma_q, gamma_k, ctx.out_ext, ctx.lse_ext, dout, window=ctx.window, **kw)
        res = {n: gr[n][:, h:].contiguous() for n in ("dq", "dg")}
    L = res["dq"].shape[1]
    dk_ext, dv_ext = gr["dk"], gr["dv"]
    if world > 1:
        acc = torch.float64 if dk_ext.dtype == torch.float64 else torch.float32
        B = dk_ext.shape[0]
        full = torch.zeros((2, B, world * L) + tuple(dk_ext.shape[2:]), dtype=acc, device=dk_ext.device)
        full[0, :, start:(rank + 1) * L] = dk_ext.to(acc)
        full[1, :, start:(rank + 1) * L] = dv_ext.to(acc)
        dist.all_reduce(full, group=group)
        mine = full[:, :, rank * L:(rank + 1) * L]
        res["dk"] = mine[0].to(dk_ext.dtype).contiguous()
        res["dv"] = mine[1].to(dv_ext.dtype).contiguous()
    else:
        res["dk"], res["dv"] = dk_ext[:, h:].contiguous(), dv_ext[:, h:].contiguous()
    dgam = torch.stack([gr["dgamma_q"], gr["dgamma_k"]]).contiguous()
    if world > 1:
        dist.all_reduce(dgam, group=group)
    res["dgamma_q"], res["dgamma_k"] = dgam[0], dgam[1]
    return res
