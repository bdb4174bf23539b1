"""GPU parity of the message block (two SO(2) convolutions with the edge-frame
activation between them) against the float64 oracle, through the C ABI.

Small and ragged graphs spanning several product tiles and chunk boundaries,
f32 (1e-4) and bf16 inputs (2e-2), forward and all eight first derivatives.
"""

import dataclasses

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


def _case(L, M, C, n, nb, seed, bf16=False):
    p = synth.make_problem("esen", seed=seed, n_atoms=n, max_nb=nb, lmax=L, mmax=M, c=C)
    rng = np.random.default_rng(seed + 50)
    w2 = rng.standard_normal(p.w.shape) * (p.w.std() if p.w.size else 1.0)
    wr2 = rng.standard_normal(p.w_rad.shape) / np.sqrt(p.n_rbf)
    b2 = rng.standard_normal(p.b_rad.shape) / np.sqrt(p.n_rbf)
    if bf16:
        p = dataclasses.replace(p, x=synth.round_bf16(p.x), w=synth.round_bf16(p.w),
                                x_bf16=True, w_bf16=True)
        w2 = synth.round_bf16(w2)
    return p, w2, wr2, b2


CASES = [
    ("L2M2C16", dict(L=2, M=2, C=16, n=80, nb=12, seed=1)),
    ("L4M2C128", dict(L=4, M=2, C=128, n=120, nb=20, seed=2)),      # ~2,400 edges, several tiles
    ("L3M1C32_chunks", dict(L=3, M=1, C=32, n=300, nb=16, seed=3)),  # crosses 2,048-edge chunks
    ("L4M2C128_bf16", dict(L=4, M=2, C=128, n=80, nb=16, seed=4, bf16=True)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_block_parity(name, kw):
    p, w2, wr2, b2 = _case(**kw)
    dt = torch.bfloat16 if p.x_bf16 else torch.float32
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    desc = B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff,
                       B.SO2_BF16 if p.x_bf16 else B.SO2_F32)
    args = (t(p.x, dt), t(p.edge_index, torch.int64), t(p.edge_vec), t(p.w, dt), t(p.w_rad),
            t(p.b_rad), t(w2, dt), t(wr2), t(b2))
    if "chunks" in name:
        B.set_max_chunk_edges(2048)
    try:
        out = B.block_forward(desc, *args)
        g = B.block_backward(desc, *args, t(p.grad_out))
        torch.cuda.synchronize()
        assert B.check(DEV) == 0
    finally:
        B.set_max_chunk_edges(0)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    oargs = (T(p.x), T(p.edge_index[0]), T(p.edge_index[1]), T(p.edge_vec), T(p.w), T(p.w_rad),
             T(p.b_rad), T(w2), T(wr2), T(b2), desc_of(p))
    tol = TOL[p.x_bf16]
    assert rel_err(out, O.block_forward(*oargs)) < tol
    ref = O.block_backward(*oargs, T(p.grad_out))
    for k in B.BLOCK_GRADS:
        assert rel_err(g[k], ref[k]) < tol, (name, k, rel_err(g[k], ref[k]))


def test_block_rejects_unequal_channels():
    desc = B.make_desc(2, 2, 16, 32, 8, 5.0)
    assert B.block_workspace_size(desc, 10, 20, 0) == 0


def test_block_lmax6_and_empty_graphs():
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    # lmax 6, mmax 3: the runtime-degree kernels and every m group
    p, w2, wr2, b2 = _case(L=6, M=3, C=32, n=60, nb=10, seed=8)
    desc = B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)
    args = (t(p.x), t(p.edge_index, torch.int64), t(p.edge_vec), t(p.w), t(p.w_rad),
            t(p.b_rad), t(w2), t(wr2), t(b2))
    out = B.block_forward(desc, *args)
    g = B.block_backward(desc, *args, t(p.grad_out))
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    oargs = (T(p.x), T(p.edge_index[0]), T(p.edge_index[1]), T(p.edge_vec), T(p.w), T(p.w_rad),
             T(p.b_rad), T(w2), T(wr2), T(b2), desc_of(p))
    assert rel_err(out, O.block_forward(*oargs)) < 1e-4
    ref = O.block_backward(*oargs, T(p.grad_out))
    for k in B.BLOCK_GRADS:
        assert rel_err(g[k], ref[k]) < 1e-4, k
    # no edges: zero output and zero gradients, nothing launched on the edges
    ei0 = torch.zeros((2, 0), dtype=torch.int64, device=DEV)
    ev0 = torch.zeros((0, 3), dtype=torch.float32, device=DEV)
    a0 = (args[0], ei0, ev0) + args[3:]
    out0 = B.block_forward(desc, *a0)
    g0 = B.block_backward(desc, *a0, t(p.grad_out))
    torch.cuda.synchronize()
    assert B.check(DEV) == 0
    assert out0.abs().max().item() == 0.0
    for k in B.BLOCK_GRADS:
        if g0[k].numel():
            assert g0[k].abs().max().item() == 0.0, k
