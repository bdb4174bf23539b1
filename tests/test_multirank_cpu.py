"""The multi-process path of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU; each rank times its own replica of the
workload and the job reports the max over ranks.  These tests run the
rendezvous, barrier and max-over-ranks helpers with world size 2 on the gloo
backend (no GPU), and check the weak-scaling arithmetic of the reported value.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import bench
    w, r, _ = bench.dist_setup()
    try:
        bench.barrier(w)
        # each rank pretends its timed region took a different time
        mine = 100.0 + 25.0 * r
        worst = bench.max_over_ranks(mine, w, torch.device("cpu"))
        q.put((r, w, worst))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_rank_rendezvous_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 for g in got)
    assert all(g[2] == pytest.approx(125.0) for g in got)


def test_weak_scaling_value():
    # value = all ranks' edges / the slowest rank's time
    world, edges, steps, worst_ms = 4, 60000, 30, 240.0
    value = world * edges * steps / (worst_ms * 1e-3)
    assert value == pytest.approx(4 * 60000 * 30 / 0.24)
