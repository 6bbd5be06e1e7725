"""bench.py's multi-rank timing on CPU with two gloo ranks: every rank ends up
with the maximum over the ranks of each figure (the job takes as long as its
slowest rank); the reference arm's non-zero ranks exit without work."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, REPO)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.max_over_ranks([10.0 + 5.0 * rank, 3.0 - rank], world, dist, "cpu")
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got in res:
        assert got == [15.0, 3.0]          # the slowest rank's figure, on every rank


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, REPO)
    import bench

    class Args:
        steps, warmup, gpus = 1, 0, 2
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""
