"""Multi-GPU harness of bench.py (replicas only: no data-path collective), on CPU with two gloo
ranks: the device-timed value is the slowest rank's, every rank agrees on it, and the whole-job
rate counts the units of all ranks; the reference arm runs on rank 0 only."""

import argparse
import datetime
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()  # the timed region is bracketed by barriers on every rank
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(ms, dist, "cpu")
        e2e = bench.max_over_ranks(3.0 * (world - rank), dist, "cpu")  # rank 0 slowest here
        dist.barrier()
        q.put((rank, m, e2e, bench.whole_job_rate(64, world, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    for _, m, e2e, rate in results:
        assert m == 15.0 and e2e == 6.0
        assert rate == pytest.approx(2 * 64 / 0.015)


def test_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.whole_job_rate(256, 1, 1000.0) == pytest.approx(256.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench

    args = argparse.Namespace(config="decode-1p5b", steps=1, warmup=3, impl="reference",
                              gpus=2, no_cpu_baseline=False, no_prefill=True)
    assert bench.run_reference(args, rank=1) is None
    assert capsys.readouterr().out == ""
