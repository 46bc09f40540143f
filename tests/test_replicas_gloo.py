"""The N>1 path of bench.py (independent replicas) on CPU with 2 gloo ranks:
the timed region is the max over ranks and the work is the sum of all ranks'."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t, u = bench.aggregate(0.5 + rank, 100.0 * (rank + 1), world)
        bench.barrier(world)
        q.put((rank, t, u))
    finally:
        dist.destroy_process_group()


def test_max_time_and_sum_of_work_over_two_ranks():
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
    for rank, t, u in res:
        assert t == pytest.approx(1.5)      # max(0.5, 1.5)
        assert u == pytest.approx(300.0)    # 100 + 200


def test_single_rank_passthrough():
    import bench
    assert bench.aggregate(0.25, 7.0, 1) == (0.25, 7.0)


def test_capacity_plan_arithmetic():
    """Conversations that fit a KV budget: 32 layers x K,V x 8 kv heads x 4096
    tokens x 128 dims x 2 bytes = 512 MiB per conversation."""
    import bench
    per, b_raw, b_comp = bench.capacity_plan(160e9, 0.7725)
    assert per == 32 * 2 * 8 * 4096 * 128 * 2 == 536870912
    assert b_raw == 298 and b_comp == int(160e9 // (536870912 * 0.7725)) == 385
    assert bench.capacity_plan(1e9, 1.0)[1:] == (1, 1)
