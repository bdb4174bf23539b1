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


class _OracleOp:
    """The per-device convolution, computed by the oracle (float64, CPU)."""

    def __init__(self, od):
        self.od = od

    def forward(self, desc, x, ei, ev, w, w_rad, b_rad):
        import oracle as O
        return O.forward(x, ei[0], ei[1], ev, w, w_rad, b_rad, self.od, n_nodes=x.shape[0])

    def backward(self, desc, x, ei, ev, w, w_rad, b_rad, G):
        import oracle as O
        return O.backward(x, ei[0], ei[1], ev, w, w_rad, b_rad, self.od, G,
                          n_nodes=x.shape[0])


_SMALL = dict(n_atoms=31, max_nb=6, lmax=2, mmax=1, c=16)


def _dst_worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import bench
    from helpers import desc_of
    from so_edge_convolution_b200 import sharded as S
    w, r, _ = bench.dist_setup()
    try:
        p = bench.dst_problem("esen", w, **_SMALL)
        sg = S.ShardedGraph(torch.from_numpy(p.edge_index), torch.from_numpy(p.edge_vec),
                            p.n_nodes, r, w)
        t = bench.dst_inputs(p, sg, torch.float64, torch.float64)
        # dst_inputs gives the GPU's f32 vectors, gate weights and grad_out;
        # the float64 comparison takes the exact values
        T = torch.from_numpy
        t["edge_vec"], t["w_rad"], t["b_rad"] = sg.edge_vec, T(p.w_rad), T(p.b_rad)
        t["grad_out"] = sg.local_rows(T(p.grad_out))
        step = bench.make_dst_step(sg, None, op=_OracleOp(desc_of(p)))
        out, g = step(t)
        q.put((r, sg.n0, sg.n1, out[: sg.n1 - sg.n0].numpy(), g["grad_x"][: sg.n1 - sg.n0].numpy(),
               sg.edge_ids.numpy(), g["grad_edge_vec"].numpy(), g["grad_w"].numpy()))
    finally:
        dist.destroy_process_group()


def test_bench_destination_split_step_on_two_ranks():
    """bench.py's --split dst step (its graph, the rank's inputs and the step
    built on so_edge_convolution_b200.sharded) on two gloo ranks, with the
    oracle standing in for the GPU convolution, equals the single-process
    result on the whole graph."""
    import numpy as np
    import bench
    from helpers import oracle_backward, oracle_forward
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dst_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    p = bench.dst_problem("esen", 2, **_SMALL)
    assert p.n_nodes == 62  # two ranks' worth of atoms
    ref_out = oracle_forward(p).numpy()
    ref = {k: v.numpy() for k, v in oracle_backward(p).items()}
    np.testing.assert_allclose(np.concatenate([r[3] for r in res]), ref_out, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(np.concatenate([r[4] for r in res]), ref["grad_x"], rtol=1e-10,
                               atol=1e-10)
    gev = np.zeros_like(ref["grad_edge_vec"])
    for r in res:
        gev[r[5]] = r[6]
        np.testing.assert_allclose(r[7], ref["grad_w"], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gev, ref["grad_edge_vec"], rtol=1e-10, atol=1e-10)


def test_dst_problem_keeps_density():
    import bench
    from so_edge_convolution_b200 import synth
    one = bench.dst_problem("esen", 1, n_atoms=200, max_nb=8, lmax=1, mmax=1, c=16)
    four = bench.dst_problem("esen", 4, n_atoms=200, max_nb=8, lmax=1, mmax=1, c=16)
    assert four.n_nodes == 4 * one.n_nodes
    d = synth.CONFIGS["esen"]["density"]
    box1, box4 = (200 / d) ** (1 / 3), (800 / d) ** (1 / 3)
    assert one.pos.max() <= box1 and four.pos.max() <= box4 and four.pos.max() > box1
    # edges per atom about the same (the neighbour cap applies to both)
    assert abs(four.n_edges / four.n_nodes - one.n_edges / one.n_nodes) < 1.0
