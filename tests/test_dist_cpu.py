"""Multi-rank bench logic on CPU (gloo, world size 2): each rank owns its own
batch (weak scaling, no collective on the data path), the step time is the max
over ranks, and the whole-job value aggregates every rank's work."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    # each rank reports a different local time; everyone must see the max
    local_ms = 10.0 + 5.0 * rank
    t = bench.max_over_ranks(local_ms, True)
    dist.barrier()
    value = bench.aggregate(2.0, world, t)
    q.put((rank, t, value))
    dist.destroy_process_group()


def test_two_ranks_take_max_time_and_aggregate_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value in res:
        assert t == 15.0                       # slowest rank
        assert value == pytest.approx(2.0 * 2 / 0.015)   # 2 ranks' work / max time


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, False) == 3.5
    assert bench.aggregate(1.0, 1, 1000.0) == pytest.approx(1.0)
