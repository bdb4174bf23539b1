"""One graph over two or three ranks (gloo, CPU): the destination-partitioned path.

so_edge_convolution_b200.sharded splits the edges by destination owner,
all-gathers node features, reduce-scatters grad_x and all-reduces the weight
gradients.  These tests run that host logic with world sizes 2 and 3, with the
float64 oracle standing in for the per-device convolution, and check that
the ranks' pieces put together equal the single-process result on the whole
graph.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


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


def _problem():
    from so_edge_convolution_b200 import synth
    # 61 nodes: not a multiple of the world size, so the last rank is padded
    return synth.make_problem("esen", seed=7, n_atoms=61, max_nb=8, lmax=2, mmax=1, c=16)


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch.distributed as dist
    from helpers import desc_of
    from so_edge_convolution_b200 import sharded as S
    dist.init_process_group("gloo")
    try:
        p = _problem()
        T = torch.from_numpy
        ei, ev = T(p.edge_index), T(p.edge_vec)
        sg = S.ShardedGraph(ei, ev, p.n_nodes)
        op = _OracleOp(desc_of(p))
        x_local = sg.local_rows(T(p.x))
        g_local = sg.local_rows(T(p.grad_out))
        out = S.forward(sg, None, x_local, T(p.w), T(p.w_rad), T(p.b_rad), op=op)
        g = S.backward(sg, None, x_local, T(p.w), T(p.w_rad), T(p.b_rad), g_local, op=op)
        q.put((rank, sg.n0, sg.n1, out[: sg.n1 - sg.n0].numpy(),
               g["grad_x"][: sg.n1 - sg.n0].numpy(), sg.edge_ids.numpy(),
               g["grad_edge_vec"].numpy(), g["grad_w"].numpy(), g["grad_w_rad"].numpy(),
               g["grad_b_rad"].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_graph_matches_single_process(world):
    from helpers import oracle_backward, oracle_forward
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    res.sort(key=lambda r: r[0])
    p = _problem()
    ref_out = oracle_forward(p).numpy()
    ref = {k: v.numpy() for k, v in oracle_backward(p).items()}
    out = np.concatenate([r[3] for r in res])
    gx = np.concatenate([r[4] for r in res])
    # contiguous node ranges covering every node once, in rank order
    assert res[0][1] == 0 and res[-1][2] == p.n_nodes
    assert all(res[k][2] == res[k + 1][1] for k in range(world - 1))
    np.testing.assert_allclose(out, ref_out, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gx, ref["grad_x"], rtol=1e-10, atol=1e-10)
    # every edge belongs to exactly one rank; its gradient lands in place
    ids = np.concatenate([r[5] for r in res])
    assert sorted(ids.tolist()) == list(range(p.n_edges))
    gev = np.zeros_like(ref["grad_edge_vec"])
    for r in res:
        gev[r[5]] = r[6]
    np.testing.assert_allclose(gev, ref["grad_edge_vec"], rtol=1e-10, atol=1e-10)
    for k, i in (("grad_w", 7), ("grad_w_rad", 8), ("grad_b_rad", 9)):
        for r in res:  # summed over ranks, the same on each
            np.testing.assert_allclose(r[i], ref[k], rtol=1e-10, atol=1e-10)


def test_node_ranges_cover_nodes_once():
    from so_edge_convolution_b200.sharded import node_range
    for n, world in ((61, 2), (100, 8), (7, 4), (5, 8)):
        seen = []
        for r in range(world):
            n0, n1, per = node_range(n, r, world)
            assert 0 <= n1 - n0 <= per and per * world >= n
            seen += list(range(n0, n1))
        assert seen == list(range(n))
