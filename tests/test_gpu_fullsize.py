"""GPU parity at the benchmark sizes, on sampled outputs and exact identities.

The full workloads (eSEN-like E = 60,000 f32; UMA-like E = 150,000 bf16;
Large E = 1,000,000 bf16) run through the C ABI in the launch configuration
bench.py times.  The float64 oracle cannot run them whole, so:

* sampled outputs it can compute one by one: out rows of sampled destination
  nodes (from their incoming edges only), grad_x rows of sampled source nodes
  (from their outgoing edges), grad_edge_vec of sampled edges, d_grad_out rows
  of sampled destinations in the double backward;
* identities that hold at any size because the map is linear in x, in the
  mixing weights and jointly in (W_rad, b):
      <grad_x, x> = <grad_w, w> = <grad_w_rad, W_rad> + <grad_b, b> = <grad_out, out>
  and, for the double backward with an edge-vector cotangent,
      <d_w, w> = <gg_r, grad_edge_vec>;
* the weight gradients element by element.  They are sums over all edges, so
  for the eSEN-like graph the oracle runs over chunks of 4,096 edges and the
  chunks' gradients are added.  For every workload a second backward takes a
  grad_out that is zero except on a few sampled destination nodes: the GPU
  still runs the whole graph in the same launch configuration (chunks and
  K-split counts depend only on the sizes), while only the sampled nodes'
  incoming edges contribute, so the oracle on those edges gives the exact
  gradients.  The force test does the same with an edge-vector cotangent that
  is zero except on sampled edges (which also gives d_edge_vec of those edges
  element by element, and zero elsewhere).
"""

import numpy as np
import pytest
import torch

import oracle as O
from so_edge_convolution_b200 import binding as B
from so_edge_convolution_b200 import synth

from helpers import desc_of, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = {False: 1e-4, True: 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from so_edge_convolution_b200 import build
    build.build()
    B.load()


def _dev(p):
    dt = torch.bfloat16 if p.x_bf16 else torch.float32
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    return dict(x=t(p.x, dt), edge_index=t(p.edge_index, torch.int64), edge_vec=t(p.edge_vec),
                w=t(p.w, dt), w_rad=t(p.w_rad), b_rad=t(p.b_rad), grad_out=t(p.grad_out))


def _bdesc(p):
    return B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff,
                       B.SO2_BF16 if p.x_bf16 else B.SO2_F32)


def _oracle_args(p, sel):
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    return (T(p.x), T(p.edge_index[0, sel]), T(p.edge_index[1, sel]), T(p.edge_vec[sel]),
            T(p.w), T(p.w_rad), T(p.b_rad), desc_of(p))


def _dot(a, b):
    return float((a.double() * b.double()).sum())


def _check_workload(name, n_nodes_sample=6, n_edges_sample=64, n_wnodes=60):
    p = synth.make_problem(name, seed=0)
    d = _dev(p)
    desc = _bdesc(p)
    out = B.forward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"])
    g = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"],
                   d["grad_out"])
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    tol = TOL[p.x_bf16]
    rng = np.random.default_rng(5)
    src, dst = p.edge_index
    # out rows of sampled destinations
    nodes = rng.choice(p.n_nodes, n_nodes_sample, replace=False)
    sel = np.nonzero(np.isin(dst, nodes))[0]
    ref = O.forward(*_oracle_args(p, sel))
    got = out.double().cpu()
    assert rel_err(got[nodes], ref[nodes]) < tol
    # grad_x rows of sampled sources and grad_edge_vec of their edges
    G = torch.from_numpy(p.grad_out)
    sel = np.nonzero(np.isin(src, nodes))[0]
    gref = O.backward(*_oracle_args(p, sel), G)
    assert rel_err(g["grad_x"].cpu()[nodes], gref["grad_x"][nodes]) < tol
    es = rng.choice(p.n_edges, n_edges_sample, replace=False)
    gref_e = O.backward(*_oracle_args(p, es), G)
    assert rel_err(g["grad_edge_vec"].cpu()[es], gref_e["grad_edge_vec"]) < tol
    # linearity identities at full size (the bf16 path rounds its tensor-core
    # operands to bf16, so the two sides agree to bf16 accuracy there)
    itol = 1e-3 if not p.x_bf16 else 1e-2
    L = _dot(d["grad_out"], out)
    wr = d["w"].float()
    assert abs(_dot(g["grad_x"], d["x"].float()) - L) < itol * abs(L) + 1e-6
    assert abs(_dot(g["grad_w"], wr) - L) < itol * abs(L) + 1e-6
    rad = _dot(g["grad_w_rad"], d["w_rad"]) + _dot(g["grad_b_rad"], d["b_rad"])
    assert abs(rad - L) < itol * abs(L) + 1e-6
    # weight gradients element by element: grad_out kept on sampled
    # destinations only, so that the oracle needs only their incoming edges
    wnodes = rng.choice(p.n_nodes, n_wnodes, replace=False)
    Gm = np.zeros_like(p.grad_out)
    Gm[wnodes] = p.grad_out[wnodes]
    gm = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                    d["b_rad"], torch.from_numpy(Gm).float().to(DEV),
                    need=["grad_w", "grad_w_rad", "grad_b_rad"])
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    sel = np.nonzero(np.isin(dst, wnodes))[0]
    wref = O.backward(*_oracle_args(p, sel), torch.from_numpy(Gm))
    for k in ("grad_w", "grad_w_rad", "grad_b_rad"):
        assert rel_err(gm[k].cpu(), wref[k]) < tol, k
    return p, d, desc, g


def _oracle_weight_grads_chunked(p, chunk=4096):
    """grad_w, grad_w_rad, grad_b_rad of the whole graph: the oracle's
    backward over consecutive edge chunks, added up (each is a sum over
    edges)."""
    G = torch.from_numpy(p.grad_out)
    acc = None
    for e0 in range(0, p.n_edges, chunk):
        sel = np.arange(e0, min(e0 + chunk, p.n_edges))
        g = O.backward(*_oracle_args(p, sel), G)
        part = {k: g[k] for k in ("grad_w", "grad_w_rad", "grad_b_rad")}
        acc = part if acc is None else {k: acc[k] + part[k] for k in acc}
    return acc


def test_esen_full_size():
    p, d, desc, g = _check_workload("esen")
    ref = _oracle_weight_grads_chunked(p)
    for k in ("grad_w", "grad_w_rad", "grad_b_rad"):
        assert rel_err(g[k].cpu(), ref[k]) < 1e-4, k


def test_uma_full_size():
    _check_workload("uma", n_nodes_sample=3, n_edges_sample=32, n_wnodes=20)


def test_large_full_size():
    _check_workload("large", n_nodes_sample=3, n_edges_sample=32, n_wnodes=40)


def test_force_double_backward_full_size():
    p = synth.make_problem("force", seed=0)
    d = _dev(p)
    desc = _bdesc(p)
    g = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"],
                   d["grad_out"], need=["grad_edge_vec"])["grad_edge_vec"]
    gg_r = torch.from_numpy(np.random.default_rng(7).standard_normal(p.edge_vec.shape)).float()
    dd = B.double_backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                           d["b_rad"], d["grad_out"], gg_edge_vec=gg_r.to(DEV))
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    # <d_w, w> = <gg_r, grad_edge_vec>: both sides linear in w
    q = _dot(gg_r, g.cpu())
    assert abs(_dot(dd["d_w"], d["w"]) - q) < 1e-3 * abs(q) + 1e-6
    # d_w, d_w_rad, d_b_rad element by element: a cotangent that is zero
    # except on 1,024 sampled edges (Q is a sum of per-edge terms, so only
    # those edges contribute), the GPU on the whole graph
    es = np.sort(np.random.default_rng(9).choice(p.n_edges, 1024, replace=False))
    ggm = torch.zeros_like(gg_r)
    ggm[es] = gg_r[es]
    dm = B.double_backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                           d["b_rad"], d["grad_out"], gg_edge_vec=ggm.to(DEV),
                           need=["d_w", "d_w_rad", "d_b_rad", "d_edge_vec"])
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    mref = O.double_backward(*_oracle_args(p, es), torch.from_numpy(p.grad_out),
                             gg_edge_vec=gg_r.double()[es])
    for k in ("d_w", "d_w_rad", "d_b_rad"):
        assert rel_err(dm[k].cpu(), mref[k]) < 1e-4, k
    # second order in the edge vectors: nonzero only on the sampled edges
    dr = dm["d_edge_vec"].cpu()
    assert rel_err(dr[es], mref["d_edge_vec"]) < 1e-4
    rest = np.setdiff1d(np.arange(p.n_edges), es)
    assert dr[rest].abs().max().item() == 0.0
    # sampled rows of d_grad_out and d_x against the oracle on the local edges
    rng = np.random.default_rng(8)
    nodes = rng.choice(p.n_nodes, 3, replace=False)
    src, dst = p.edge_index
    for key, row, sel in (("d_grad_out", dst, np.nonzero(np.isin(dst, nodes))[0]),
                          ("d_x", src, np.nonzero(np.isin(src, nodes))[0])):
        args = _oracle_args(p, sel)
        ref = O.double_backward(*args, torch.from_numpy(p.grad_out),
                                gg_edge_vec=gg_r.double()[sel])
        assert rel_err(dd[key].cpu()[nodes], ref[key][nodes]) < 1e-4, key


@pytest.mark.parametrize("L,M,C", [(6, 6, 64), (3, 2, 256), (6, 2, 512)])
def test_extreme_shapes(L, M, C):
    # largest lmax and mmax, and the widest channel counts, on a small graph
    from helpers import oracle_backward, oracle_forward
    p = synth.make_problem("esen", seed=3, n_atoms=40, max_nb=6, lmax=L, mmax=M, c=C)
    d = _dev(p)
    desc = _bdesc(p)
    out = B.forward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"])
    g = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"],
                   d["grad_out"])
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    assert rel_err(out, oracle_forward(p)) < 1e-4
    ref = oracle_backward(p)
    for k in ["grad_x", "grad_w", "grad_w_rad", "grad_b_rad", "grad_edge_vec"]:
        assert rel_err(g[k], ref[k]) < 1e-4, k
