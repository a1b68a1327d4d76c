"""Multi-rank host logic of bench.py, run as world_size-2 gloo process groups on the CPU.

The layer shards by sequence: every rank runs its own independent batch and the ranks
exchange nothing but the timing reduction.  These tests check that reduction (max over
ranks, delivered to every rank), the whole-job throughput built on it, that the ranks draw
different batches, and that the reference arm does no work on ranks other than 0.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    from global_attention_b200.synth import make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        assert (w, r, lr) == (world, rank, rank)

        # every rank receives the largest time, whatever order the ranks report in
        t_rank = 10.0 + 3.5 * rank
        t_max = bench.max_over_ranks(t_rank, world, "cpu")
        assert t_max == 10.0 + 3.5 * (world - 1)

        # weak scaling: tokens of all ranks over the slowest rank's step
        tokens = 4 * 16384
        assert bench.job_throughput(tokens, world, t_max) == pytest.approx(tokens * world / (t_max / 1e3))

        # independent batches: each rank's inputs differ from every other rank's
        t = make_inputs(1, 64, seed=bench.rank_seed(rank), with_dout=True)
        digest = float(t["q"].float().sum() + 2 * t["k"].float().sum() + 3 * t["dout"].float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        assert len(set(digests)) == world

        # the bench's barrier -> work -> barrier bracket: the reported time covers the slowest rank
        import time
        dist.barrier()
        t0 = time.perf_counter()
        time.sleep(0.05 * (rank + 1))
        el = (time.perf_counter() - t0) * 1e3
        dist.barrier()
        reported = bench.max_over_ranks(el, world, "cpu")
        assert reported >= 0.05 * world * 1e3 * 0.9
        results[rank] = reported
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
    assert len(results) == world
    assert results[0] == results[1]          # one number for the job, the same on every rank


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.25, 1, "cpu") == 7.25
    assert bench.job_throughput(65536, 1, 3.5) == pytest.approx(65536 / 3.5e-3)
    assert bench.job_throughput(65536, 8, 3.5) == pytest.approx(8 * 65536 / 3.5e-3)
    assert len({bench.rank_seed(r) for r in range(8)}) == 8


def test_reference_arm_idle_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
