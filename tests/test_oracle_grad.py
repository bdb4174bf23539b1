"""Pins for the oracle's backward and double backward (no GPU).

Central finite differences (h = 1e-6, float64) of the scalar
<grad_out, forward(...)> and of Q = <gg_x, grad_x> + <gg_r, grad_edge_vec>
against the autograd results, on tiny random graphs; plus the rotation
invariance of an l = 0 energy (zero net torque on the edge vectors).
"""

import numpy as np
import pytest
import torch

import oracle as O
from so_edge_convolution_b200 import synth

T = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.float64)  # noqa: E731
I64 = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.int64)  # noqa: E731
H = 1e-6


def _setup(L=2, M=2, ci=2, co=3, n=5, e=12, seed=0):
    p = synth.random_graph(n, e, L, M, ci, co, seed=seed)
    desc = O.Desc(L, M, ci, co, p.n_rbf, p.rbf_cutoff)
    args = dict(x=T(p.x), w=T(p.w), w_rad=T(p.w_rad), b_rad=T(p.b_rad),
                edge_vec=T(p.edge_vec))
    return p, desc, args


def _fwd(p, desc, a):
    return O.forward(a["x"], I64(p.edge_index[0]), I64(p.edge_index[1]),
                     a["edge_vec"], a["w"], a["w_rad"], a["b_rad"], desc)


def _fd(fun, t, idx):
    t = t.clone()
    flat = t.view(-1)
    old = flat[idx].item()
    flat[idx] = old + H
    fp = fun(t)
    flat[idx] = old - H
    fm = fun(t)
    return (fp - fm) / (2 * H)


def _sample(t, k, seed):
    rng = np.random.default_rng(seed)
    return rng.choice(t.numel(), size=min(k, t.numel()), replace=False)


@pytest.mark.parametrize("L,M", [(2, 2), (2, 1), (3, 2)])
def test_backward_matches_finite_differences(L, M):
    p, desc, a = _setup(L=L, M=M, seed=L + M)
    G = T(p.grad_out)
    g = O.backward(a["x"], I64(p.edge_index[0]), I64(p.edge_index[1]),
                   a["edge_vec"], a["w"], a["w_rad"], a["b_rad"], desc, G)
    names = {"x": "grad_x", "w": "grad_w", "w_rad": "grad_w_rad",
             "b_rad": "grad_b_rad", "edge_vec": "grad_edge_vec"}
    for k, gname in names.items():
        for i in _sample(a[k], 12, 7):
            def f(t, k=k):
                b = dict(a)
                b[k] = t
                return float((G * _fwd(p, desc, b)).sum())
            fd = _fd(f, a[k], i)
            an = g[gname].reshape(-1)[i].item()
            assert abs(fd - an) < 1e-7 * max(1.0, abs(an)), (k, i, fd, an)


@pytest.mark.parametrize("with_gx", [False, True])
def test_double_backward_matches_finite_differences(with_gx):
    p, desc, a = _setup(L=2, M=2, ci=2, co=2, n=4, e=10, seed=21)
    rng = np.random.default_rng(3)
    G = T(p.grad_out)
    gg_r = T(rng.standard_normal(p.edge_vec.shape))
    gg_x = T(rng.standard_normal(p.x.shape)) if with_gx else None
    src, dst = I64(p.edge_index[0]), I64(p.edge_index[1])
    d = O.double_backward(a["x"], src, dst, a["edge_vec"], a["w"], a["w_rad"],
                          a["b_rad"], desc, G, gg_x=gg_x, gg_edge_vec=gg_r)

    def q(b, Gv):
        g = O.backward(b["x"], src, dst, b["edge_vec"], b["w"], b["w_rad"],
                       b["b_rad"], desc, Gv)
        v = float((gg_r * g["grad_edge_vec"]).sum())
        if gg_x is not None:
            v += float((gg_x * g["grad_x"]).sum())
        return v

    targets = {"x": "d_x", "w": "d_w", "w_rad": "d_w_rad", "b_rad": "d_b_rad",
               "edge_vec": "d_edge_vec"}
    for k, dname in targets.items():
        for i in _sample(a[k], 8, 11):
            def f(t, k=k):
                b = dict(a)
                b[k] = t
                return q(b, G)
            fd = _fd(f, a[k], i)
            an = d[dname].reshape(-1)[i].item()
            assert abs(fd - an) < 2e-6 * max(1.0, abs(an)), (k, i, fd, an)
    for i in _sample(G, 8, 12):
        fd = _fd(lambda t: q(a, t), G, i)
        an = d["d_grad_out"].reshape(-1)[i].item()
        assert abs(fd - an) < 2e-6 * max(1.0, abs(an)), ("G", i, fd, an)


def test_energy_of_scalar_features_has_no_torque():
    # E = sum of l = 0 outputs is rotation invariant when x has only l = 0
    # content, so sum_e r_e x dE/dr_e = 0.
    p, desc, a = _setup(L=3, M=2, ci=3, co=3, n=6, e=20, seed=31)
    x = a["x"].clone()
    x[:, 1:, :] = 0
    G = torch.zeros(p.n_nodes, desc.s, desc.c_out, dtype=torch.float64)
    G[:, 0, :] = 1.0
    g = O.backward(x, I64(p.edge_index[0]), I64(p.edge_index[1]),
                   a["edge_vec"], a["w"], a["w_rad"], a["b_rad"], desc, G)
    torque = torch.cross(a["edge_vec"], g["grad_edge_vec"], dim=-1).sum(0)
    assert torque.abs().max() < 1e-12
    assert g["grad_edge_vec"].abs().max() > 1e-3  # not trivially zero
