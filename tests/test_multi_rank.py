"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Each rank compresses an independent layer (weak scaling, no data-path
collective); the job's step time is the maximum over ranks and the throughput
counts every rank's tokens.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 1.0 + 2.0 * rank                  # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, world)
        out[rank] = (bench.replica_layer(rank), job_ms, bench.job_throughput(world, 32768, job_ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_time_and_count_all_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert sorted(v[0] for v in res.values()) == [0, 1]          # independent layers
    assert all(v[1] == pytest.approx(3.0) for v in res.values())  # max over ranks
    assert all(v[2] == pytest.approx(2 * 32768 / 3e-3 / 1e6) for v in res.values())


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_throughput(1, 1000, 1.0) == pytest.approx(1.0)

