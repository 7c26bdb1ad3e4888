"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo (127.0.0.1).

Each rank is an independent replica (weak scaling, no data-path collective); the step time that
is reported is the slowest rank's, and the whole-job rate counts every rank's work.  Also checks
that the reference arm does nothing on ranks other than 0.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 2.0 + 3.0 * rank  # rank 1 is the slow one
        t = bench.max_over_ranks(local_ms, ws, torch.device("cpu"))
        rate = bench.whole_job_rate(1e12, ws, t, 1e12)
        env = bench.dist_env()

        class Args:
            steps, warmup, gpus, ref_pairs = 1, 3, ws, 8

        ref_rc = bench.run_reference(Args()) if rank != 0 else None
        q.put((rank, t, rate, env, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_the_whole_job():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, rate, env, ref_rc in results:
        assert t == 5.0                               # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 1e12 / 5e-3 / 1e12)  # both ranks' work over the slowest time
        assert env == (ws, rank, rank)
        if rank != 0:
            assert ref_rc == 0                        # the reference arm runs on rank 0 only


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(2e12, 1, 4.0, 1e12) == pytest.approx(500.0)
