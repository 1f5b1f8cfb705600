"""The N > 1 path of bench.py on CPU: world-size-2 gloo process groups.

bench.py runs N independent replicas (one process per GPU, launched by torch.distributed.run).
Its host-side plumbing is checked here without a GPU: the process group comes up, the ranks meet
at a barrier, the job time is the max over ranks, the whole-job rate counts every rank's units,
and in the reference arm only rank 0 works and prints.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    ms, value = bench.job_throughput(d, 10.0 + rank, 320)
    d.barrier()
    d.close()
    q.put((rank, ms, value))


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, value in got:
        assert ms == pytest.approx(11.0)                       # max over ranks
        assert value == pytest.approx(2 * 320 / 11.0e-3)       # units of both ranks / job time


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        d.init("gloo")   # no process group for one rank
        assert d.pg is None
        assert bench.job_throughput(d, 4.0, 64) == (4.0, 64 / 4.0e-3)


def test_reference_arm_other_ranks_do_no_work(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Rank1:
        rank, world, local = 1, 2, 1

    class Args:
        steps, warmup = 3, 3

    assert bench.run_reference(Args(), Rank1()) is None
    assert capsys.readouterr().out == ""
