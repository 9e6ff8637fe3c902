"""Multi-process rank logic on CPU (gloo, world size 2): barrier, max over ranks, per-rank
seeds and the whole-job throughput used by bench.py."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from gated_deltanet_dual_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, lr = replicas.env_rank()
    replicas.init(w, backend="gloo", timeout_s=60)
    replicas.barrier(w)
    elapsed = 10.0 + 5.0 * r                 # rank 1 is the slow one
    mx = replicas.max_over_ranks(elapsed, w)
    q.put((r, mx, replicas.replica_seed(7, r), replicas.throughput(1000, w, 4, mx)))
    replicas.shutdown(w)


def test_two_rank_max_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [x[1] for x in res] == [15.0, 15.0]          # max over ranks, same on every rank
    assert [x[2] for x in res] == [7, 8]                 # independent seeded replicas
    assert res[0][3] == pytest.approx(1000 * 2 * 4 / 0.015)


def test_single_process_defaults():
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.throughput(10, 1, 2, 1000.0) == pytest.approx(20.0)
