"""Pins of the message-block oracle (oracle/block.py).

A hand-derived two-edge case (tests/golden/block_cases.json), equivariance
under a global rotation, independence of the edge frame's roll, the lmax = 0
case written out as a gated two-layer perceptron message, and central finite
differences of every first derivative.
"""

import json
import os

import numpy as np
import pytest
import torch
from scipy.spatial.transform import Rotation

import oracle as O
from so_edge_convolution_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
T = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.float64)  # noqa: E731
I64 = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.int64)  # noqa: E731


def _problem(L=2, M=1, C=3, n=7, nb=5, seed=0):
    p = synth.make_problem("esen", seed=seed, n_atoms=n, max_nb=nb, lmax=L, mmax=M, c=C)
    rng = np.random.default_rng(seed + 100)
    w2 = rng.standard_normal(p.w.shape) / np.sqrt(3.0)
    wr2 = rng.standard_normal(p.w_rad.shape) / 4.0
    b2 = rng.standard_normal(p.b_rad.shape) / 4.0
    return p, w2, wr2, b2


def _fwd(p, w2, wr2, b2, x=None, vec=None, roll=None):
    desc = O.Desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)
    return O.block_forward(T(p.x if x is None else x), I64(p.edge_index[0]),
                           I64(p.edge_index[1]), T(p.edge_vec if vec is None else vec),
                           T(p.w), T(p.w_rad), T(p.b_rad), T(w2), T(wr2), T(b2), desc, roll=roll)


def test_hand_derived_block_case():
    with open(os.path.join(HERE, "golden", "block_cases.json")) as f:
        case = json.load(f)["cases"][0]
    desc = O.Desc(case["lmax"], case["mmax"], case["c"], case["c"], case["n_rbf"], case["cutoff"])
    ei = I64(case["edge_index"])
    out = O.block_forward(T(case["x"])[..., None], ei[0], ei[1], T(case["edge_vec"]),
                          T(case["w1"]), T(case["w_rad1"]), T(case["b_rad1"]), T(case["w2"]),
                          T(case["w_rad2"]), T(case["b_rad2"]), desc)
    expect = T(case["out"])
    assert (out[..., 0] - expect).abs().max().item() <= 1e-13 * expect.abs().max().item()


def test_block_is_rotation_equivariant():
    p, w2, wr2, b2 = _problem()
    Q = Rotation.random(random_state=3).as_matrix()
    D = O.wigner_d(torch.as_tensor(Q)[None], p.lmax)[0].numpy()
    ref = _fwd(p, w2, wr2, b2).numpy()
    rot = _fwd(p, w2, wr2, b2, x=np.einsum("st,ntc->nsc", D, p.x), vec=p.edge_vec @ Q.T).numpy()
    want = np.einsum("st,ntc->nsc", D, ref)
    assert np.abs(rot - want).max() < 1e-10 * max(1.0, np.abs(want).max())
    assert np.abs(ref).max() > 1e-3


def test_block_does_not_depend_on_the_frame_roll():
    p, w2, wr2, b2 = _problem(L=3, M=2, C=2, seed=1)
    ref = _fwd(p, w2, wr2, b2)
    roll = T(np.random.default_rng(4).uniform(0, 2 * np.pi, p.n_edges))
    assert (_fwd(p, w2, wr2, b2, roll=roll) - ref).abs().max() < 1e-12 * ref.abs().max()


def test_lmax0_block_is_a_gated_two_layer_message():
    # lmax 0: D = 1, so out[d] = sum_e g2 * (W2 (h * sigmoid(h))), h = g1 * (W1 x[s])
    p, w2, wr2, b2 = _problem(L=0, M=0, C=4, n=9, nb=6, seed=2)
    desc = O.Desc(0, 0, 4, 4, p.n_rbf, p.rbf_cutoff)
    got = _fwd(p, w2, wr2, b2).numpy()[:, 0, :]
    d = T(np.linalg.norm(p.edge_vec, axis=1))
    g1 = O.gate(d, T(p.w_rad), T(p.b_rad), desc).numpy()
    g2 = O.gate(d, T(wr2), T(b2), desc).numpy()
    W1, W2 = p.w.reshape(4, 4), w2.reshape(4, 4)
    want = np.zeros((p.n_nodes, 4))
    for e in range(p.n_edges):
        s, t = p.edge_index[:, e]
        h = g1[e] * (W1 @ p.x[s, 0])
        want[t] += g2[e] * (W2 @ (h / (1.0 + np.exp(-h))))
    assert np.abs(got - want).max() < 1e-12 * np.abs(want).max()


def test_block_backward_matches_finite_differences():
    p, w2, wr2, b2 = _problem(L=2, M=1, C=2, n=5, nb=4, seed=5)
    desc = O.Desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)
    G = T(np.random.default_rng(6).standard_normal(p.x.shape))
    args = [T(p.x), T(p.w), T(p.w_rad), T(p.b_rad), T(w2), T(wr2), T(b2), T(p.edge_vec)]
    src, dst = I64(p.edge_index[0]), I64(p.edge_index[1])

    def loss(a):
        x, w1, r1, c1, ww2, r2, c2, vec = a
        return float((G * O.block_forward(x, src, dst, vec, w1, r1, c1, ww2, r2, c2, desc)).sum())

    g = O.block_backward(*args[:7][:1], src, dst, args[7], *args[1:7], desc, G)
    names = dict(zip(range(8), ["grad_x", "grad_w1", "grad_w_rad1", "grad_b_rad1", "grad_w2",
                                "grad_w_rad2", "grad_b_rad2", "grad_edge_vec"]))
    rng = np.random.default_rng(7)
    h = 1e-6
    for i, name in names.items():
        flat = args[i].reshape(-1)
        for j in rng.choice(flat.numel(), min(6, flat.numel()), replace=False):
            plus = [a.clone() for a in args]
            minus = [a.clone() for a in args]
            plus[i].reshape(-1)[j] += h
            minus[i].reshape(-1)[j] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = float(g[name].reshape(-1)[j])
            assert abs(fd - an) < 1e-6 * max(1.0, abs(an)), (name, j, fd, an)
