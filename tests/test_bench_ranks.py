"""bench.py's multi-rank path on CPU with two gloo ranks: the job time is the
max over ranks and the throughput counts every rank's work (replicas, weak
scaling); the reference arm's non-zero ranks exit without work."""
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
    ms_per_step, per_s = bench.aggregate_over_ranks(10.0 + 5.0 * rank, 5, 1.0e12, world, dist, "cpu")
    q.put((rank, ms_per_step, per_s))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_all_work():
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
    for rank, ms_per_step, per_s in res:
        assert ms_per_step == pytest.approx(15.0 / 5)            # max over ranks: 15 ms for 5 steps
        assert per_s == pytest.approx(2 * 1.0e12 * 5 / 0.015)   # both ranks' work over the max time


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, REPO)
    import bench

    class Args:
        steps, warmup, gpus = 1, 0, 2
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""
