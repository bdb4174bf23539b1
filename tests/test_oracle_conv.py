"""Pins for the oracle's forward map (no GPU).

Hand-derived golden cases, a brute-force second formulation, equivariance,
invariance of l = 0 outputs, roll invariance, the lmax = 0 textbook case, a
direction-independent special case and an exact integer reduction test.
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


def _run(p, desc=None, **kw):
    desc = desc or O.Desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf,
                          p.rbf_cutoff)
    return O.forward(T(p.x), I64(p.edge_index[0]), I64(p.edge_index[1]),
                     T(p.edge_vec), T(p.w), T(p.w_rad), T(p.b_rad), desc, **kw)


def _hand_cases():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: c["name"])
def test_hand_derived_cases(case):
    desc = O.Desc(case["lmax"], case["mmax"], case["c"], case["c"],
                  case["n_rbf"], case["cutoff"])
    x = T(case["x"])[..., None]
    ei = I64(case["edge_index"])
    out = O.forward(x, ei[0], ei[1], T(case["edge_vec"]), T(case["w"]),
                    T(case["w_rad"]), T(case["b_rad"]), desc)
    expect = T(case["out"])
    # the oracle's D comes from a least-squares fit (rounding ~1e-15 relative)
    tol = 1e-13 * max(1.0, expect.abs().max().item())
    assert (out[..., 0] - expect).abs().max().item() <= tol


@pytest.mark.parametrize("L,M,ci,co", [(2, 2, 2, 3), (3, 1, 2, 2), (2, 0, 1, 2)])
def test_batched_matches_per_edge_loop(L, M, ci, co):
    p = synth.random_graph(6, 14, L, M, ci, co, seed=L * 10 + M)
    desc = O.Desc(L, M, ci, co, p.n_rbf, p.rbf_cutoff)
    a = _run(p, desc)
    b = O.forward_loop(T(p.x), I64(p.edge_index[0]), I64(p.edge_index[1]),
                       T(p.edge_vec), T(p.w), T(p.w_rad), T(p.b_rad), desc)
    assert (a - b).abs().max() < 1e-12 * max(1.0, b.abs().max().item())


def _rotate_problem(p, Q):
    """Rotate every edge vector by Q and every feature by D(Q)."""
    D = O.wigner_d(torch.as_tensor(Q)[None], p.lmax)[0].numpy()
    x = np.einsum("st,ntc->nsc", D, p.x)
    vec = p.edge_vec @ Q.T
    import dataclasses
    return dataclasses.replace(p, x=x, edge_vec=vec), D


@pytest.mark.parametrize("name", ["tiny"])
def test_equivariance(name):
    p = synth.make_problem(name)
    Q = Rotation.random(random_state=11).as_matrix()
    q, D = _rotate_problem(p, Q)
    out = _run(p).numpy()
    out_q = _run(q).numpy()
    expect = np.einsum("st,ntc->nsc", D, out)
    assert np.abs(out_q - expect).max() < 1e-10 * max(1, np.abs(out).max())
    # l = 0 rows do not move at all
    assert np.abs(out_q[:, 0] - out[:, 0]).max() < 1e-10 * max(
        1, np.abs(out).max())


def test_roll_invariance():
    p = synth.random_graph(7, 20, 3, 2, 3, 2, seed=5)
    base = _run(p)
    roll = T(np.random.default_rng(2).uniform(-np.pi, np.pi, p.n_edges))
    rolled = _run(p, roll=roll)
    assert (base - rolled).abs().max() < 1e-12 * max(1, base.abs().max())


def test_roll_changes_the_edge_frame_coefficients():
    # Control for the test above: the roll hook does change the edge-frame
    # coefficients (the m = +1 row of l = 1), only the output is roll-free.
    p = synth.random_graph(5, 10, 2, 2, 2, 2, seed=6)
    roll = T(np.random.default_rng(3).uniform(0.5, 2.5, p.n_edges))
    vec = T(p.edge_vec)
    R = O.frame(vec / vec.norm(dim=-1, keepdim=True))
    D = O.wigner_d_blocks(R, 1)[1]
    Dr = O.wigner_d_blocks(torch.einsum("eij,ejk->eik", _rz(roll), R), 1)[1]
    xs = T(p.x)[I64(p.edge_index[0]), 1:4, 0]
    c0 = torch.einsum("ej,ej->e", D[:, 2], xs)
    c1 = torch.einsum("ej,ej->e", Dr[:, 2], xs)
    assert (c0 - c1).abs().max() > 1e-3


def _rz(a):
    c, s = torch.cos(a), torch.sin(a)
    o, z = torch.ones_like(c), torch.zeros_like(c)
    return torch.stack([torch.stack([c, -s, z], -1), torch.stack([s, c, z], -1),
                        torch.stack([z, z, o], -1)], -2)


def test_lmax0_is_gather_gemm_scatter():
    p = synth.random_graph(9, 30, 0, 0, 4, 5, seed=8)
    out = _run(p).numpy()
    d = np.linalg.norm(p.edge_vec, axis=1)
    mu = np.linspace(0, p.rbf_cutoff, p.n_rbf)
    sig = p.rbf_cutoff / (p.n_rbf - 1)
    phi = np.exp(-(d[:, None] - mu[None]) ** 2 / (2 * sig * sig))
    g = phi @ p.w_rad + p.b_rad
    W0 = p.w.reshape(p.c_out, p.c_in)
    y = g * (p.x[p.edge_index[0], 0, :] @ W0.T)
    expect = np.zeros((p.n_nodes, 1, p.c_out))
    np.add.at(expect[:, 0, :], p.edge_index[1], y)
    assert np.abs(out - expect).max() < 1e-12


def test_direction_independent_special_case():
    # mmax = lmax, W0 = blockdiag_l(W_l), W1_m = blockdiag_{l>=m}(W_l),
    # W2 = 0  =>  out[d] += g * W_l x[s]_l, whatever the edge direction.
    L, ci, co = 3, 2, 3
    p = synth.random_graph(6, 16, L, L, ci, co, seed=9)
    rng = np.random.default_rng(10)
    Wl = [rng.standard_normal((co, ci)) for _ in range(L + 1)]
    W0 = np.zeros(((L + 1) * co, (L + 1) * ci))
    for l in range(L + 1):
        W0[l * co:(l + 1) * co, l * ci:(l + 1) * ci] = Wl[l]
    blocks = [W0.reshape(-1)]
    for m in range(1, L + 1):
        k = L + 1 - m
        W1 = np.zeros((k * co, k * ci))
        for l in range(m, L + 1):
            W1[(l - m) * co:(l - m + 1) * co, (l - m) * ci:(l - m + 1) * ci] = Wl[l]
        blocks += [W1.reshape(-1), np.zeros(k * co * k * ci)]
    import dataclasses
    q = dataclasses.replace(p, w=np.concatenate(blocks))
    out = _run(q).numpy()
    d = np.linalg.norm(p.edge_vec, axis=1)
    mu = np.linspace(0, p.rbf_cutoff, p.n_rbf)
    sig = p.rbf_cutoff / (p.n_rbf - 1)
    g = np.exp(-(d[:, None] - mu[None]) ** 2 / (2 * sig * sig)) @ p.w_rad + p.b_rad
    expect = np.zeros((p.n_nodes, (L + 1) ** 2, co))
    xs = p.x[p.edge_index[0]]
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) ** 2)
        y = g[:, None, :] * np.einsum("oc,esc->eso", Wl[l], xs[:, sl, :])
        np.add.at(expect[:, sl, :], p.edge_index[1], y)
    assert np.abs(out - expect).max() < 1e-12


def _reduction_problem(n_nodes=40, n_edges=300, seed=12):
    p = synth.random_graph(n_nodes, n_edges, 2, 2, 4, 4, seed=seed)
    x = np.zeros_like(p.x)
    x[:, 0, :] = np.arange(n_nodes)[:, None]
    blocks = []
    for r, k in synth.weight_block_shapes(2, 2, 4, 4):
        blocks.append(np.zeros(r * k))
    W0 = np.zeros((3 * 4, 3 * 4))
    W0[:4, :4] = np.eye(4)
    blocks[0] = W0.reshape(-1)
    import dataclasses
    return dataclasses.replace(p, x=x, w=np.concatenate(blocks),
                               w_rad=np.zeros_like(p.w_rad),
                               b_rad=np.ones_like(p.b_rad))


def test_reduction_set_is_exact():
    p = _reduction_problem()
    out = _run(p).numpy()
    expect = np.bincount(p.edge_index[1], weights=p.edge_index[0],
                         minlength=p.n_nodes)
    assert np.array_equal(out[:, 0, 0], expect)
    assert np.all(out[:, 1:, :] == 0)


def test_empty_graph_and_isolated_nodes():
    p = synth.random_graph(4, 0, 2, 1, 2, 2, seed=13)
    out = _run(p)
    assert out.shape == (4, 9, 2) and float(out.abs().max()) == 0.0
    q = synth.random_graph(6, 5, 2, 1, 2, 2, seed=14)
    out = _run(q).numpy()
    cold = sorted(set(range(6)) - set(q.edge_index[1].tolist()))
    assert cold and np.all(out[cold] == 0)


def test_zero_length_edge_is_rejected():
    p = synth.random_graph(3, 2, 1, 1, 1, 1, seed=15)
    p.edge_vec[1] = 0.0
    with pytest.raises(ValueError):
        _run(p)


def _wrong_width(d, desc):
    mu = torch.linspace(0.0, desc.cutoff, desc.n_rbf, dtype=d.dtype)
    sigma = desc.cutoff / desc.n_rbf
    return torch.exp(-((d[:, None] - mu[None, :]) ** 2) / (2.0 * sigma * sigma))


def _wrong_centres(d, desc):
    sigma = desc.cutoff / (desc.n_rbf - 1)
    mu = torch.arange(desc.n_rbf, dtype=d.dtype) * (desc.cutoff / desc.n_rbf)
    return torch.exp(-((d[:, None] - mu[None, :]) ** 2) / (2.0 * sigma * sigma))


@pytest.mark.parametrize("planted", [_wrong_width, _wrong_centres], ids=["width", "centres"])
def test_radial_case_catches_a_planted_basis_mistake(planted, monkeypatch):
    """The radial-gate hand case fails if the oracle's Gaussian basis used
    another width or other centres (the mistake is planted in the oracle)."""
    import oracle.so2conv as S
    case = [c for c in _hand_cases() if c["name"] == "radial_gate_on_centres"][0]
    monkeypatch.setattr(S, "rbf", planted)
    desc = O.Desc(case["lmax"], case["mmax"], case["c"], case["c"], case["n_rbf"], case["cutoff"])
    ei = I64(case["edge_index"])
    out = O.forward(T(case["x"])[..., None], ei[0], ei[1], T(case["edge_vec"]), T(case["w"]),
                    T(case["w_rad"]), T(case["b_rad"]), desc)
    assert (out[..., 0] - T(case["out"])).abs().max().item() > 1e-3
