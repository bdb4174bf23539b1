"""One graph split by destination over ranks, on one GPU.

The per-rank convolutions run through the C ABI on cuda:0.  Two ranks are
emulated by running each rank's edge share in turn and combining on the host
(no rank waits on another), and the collectives themselves run through NCCL
with a single rank.  Both are checked against the float64 oracle on the whole
graph, with the parity tolerances of the unsharded path.
"""

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from so_edge_convolution_b200 import binding as B
from so_edge_convolution_b200 import sharded as S
from so_edge_convolution_b200 import synth

from helpers import oracle_backward, oracle_forward, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = {False: 1e-4, True: 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from so_edge_convolution_b200 import build
    build.build()
    B.load()
    torch.cuda.init()


def _problem(bf16):
    p = synth.make_problem("uma" if bf16 else "esen", seed=11, n_atoms=301, max_nb=16,
                           lmax=3, mmax=2, c=64)
    return p


def _tensors(p):
    dt = torch.bfloat16 if p.x_bf16 else torch.float32
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    desc = B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff,
                       B.SO2_BF16 if p.x_bf16 else B.SO2_F32)
    return desc, dict(x=t(p.x, dt), ei=t(p.edge_index, torch.int64), ev=t(p.edge_vec),
                      w=t(p.w, dt), wr=t(p.w_rad), br=t(p.b_rad), G=t(p.grad_out))


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_two_rank_shares_assemble_to_the_whole_graph(bf16):
    p = _problem(bf16)
    desc, d = _tensors(p)
    N, world = p.n_nodes, 2
    ref_out = oracle_forward(p)
    ref = oracle_backward(p)
    out = torch.zeros((N,) + tuple(ref_out.shape[1:]), dtype=torch.float64)
    gx = torch.zeros_like(ref["grad_x"])
    gev = torch.zeros_like(ref["grad_edge_vec"])
    gw = {k: 0.0 for k in ("grad_w", "grad_w_rad", "grad_b_rad")}
    seen = []
    for rank in range(world):
        sg = S.ShardedGraph(d["ei"], d["ev"], N, rank=rank, world=world)
        x_full = torch.zeros((sg.n_pad,) + tuple(d["x"].shape[1:]), dtype=d["x"].dtype,
                             device=DEV)
        x_full[:N] = d["x"]
        o = B.forward(desc, x_full, sg.edge_index, sg.edge_vec, d["w"], d["wr"], d["br"])
        g_full = torch.zeros((sg.n_pad,) + tuple(d["G"].shape[1:]), device=DEV)
        g_full[sg.n0:sg.n1] = d["G"][sg.n0:sg.n1]
        g = B.backward(desc, x_full, sg.edge_index, sg.edge_vec, d["w"], d["wr"], d["br"],
                       g_full)
        assert B.check(DEV) == 0
        out[sg.n0:sg.n1] = o[sg.n0:sg.n1].double().cpu()
        # rows outside the rank's range get no edge, so they stay zero
        assert not o[:sg.n0].any() and not o[sg.n1:].any()
        gx += g["grad_x"][:N].double().cpu()
        gev[sg.edge_ids.cpu()] = g["grad_edge_vec"].double().cpu()
        for k in gw:
            gw[k] = gw[k] + g[k].double().cpu()
        seen += sg.edge_ids.tolist()
    assert sorted(seen) == list(range(p.n_edges))
    tol = TOL[bf16]
    assert rel_err(out, ref_out) < tol
    assert rel_err(gx, ref["grad_x"]) < tol
    assert rel_err(gev, ref["grad_edge_vec"]) < tol
    for k in gw:
        assert rel_err(gw[k], ref[k]) < tol, k


def test_nccl_collectives_single_rank():
    p = _problem(False)
    desc, d = _tensors(p)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device(DEV))
    try:
        sg = S.ShardedGraph(d["ei"], d["ev"], p.n_nodes)
        assert (sg.n0, sg.n1) == (0, p.n_nodes) and sg.edge_ids.numel() == p.n_edges
        out = S.forward(sg, desc, sg.local_rows(d["x"]), d["w"], d["wr"], d["br"])
        g = S.backward(sg, desc, sg.local_rows(d["x"]), d["w"], d["wr"], d["br"],
                       sg.local_rows(d["G"]))
        torch.cuda.synchronize()
        assert B.check(DEV) == 0
    finally:
        dist.destroy_process_group()
    ref_out = oracle_forward(p)
    ref = oracle_backward(p)
    assert rel_err(out[:p.n_nodes], ref_out) < TOL[False]
    for k in ("grad_x",):
        assert rel_err(g[k][:p.n_nodes], ref[k]) < TOL[False]
    for k in ("grad_w", "grad_w_rad", "grad_b_rad", "grad_edge_vec"):
        assert rel_err(g[k], ref[k]) < TOL[False], k
