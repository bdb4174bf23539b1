"""The message block: two SO(2) convolutions with the activation between them
(oracle, float64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"TrimSO(2): Fast and Memory-Efficient Training of Equivariant Interatomic
Potentials" (Abstract) names three fused stages of an SO(2) model's dataflow:
rotation on gather, recombination with activation, and inverse rotation on
reduction.  The activation sits between the two dense SO(2) multiplications
of a message block, in the edge frame.  The page prints no formula; this is
the reading (all channel counts equal, C):

    a   = trunc(D(R_e) x[s])                      rotation on gather
    h   = g1(|r_e|) * M_W1(a)                     first SO(2) conv, gated
    h'  = h * sigmoid(h[(0,0)])                   activation, per channel
    y~  = g2(|r_e|) * M_W2(h')                    second SO(2) conv, gated
    out[d] += D(R_e)^T y~                         inverse rotation on reduction

On the (0, 0) row the activation is SiLU; every other row of a channel is
gated by the sigmoid of that channel's (0, 0) value.  h[(0,0)] is unchanged
by a roll of the edge frame about z_hat, so the activation commutes with the
roll and the block is rotation-equivariant like the single convolution.  M_W is the per-m mixing of the single convolution (W0 on the
m = 0 rows, the (W1_m, W2_m) pair map on +-m), each conv with its own packed
weights and radial gate.
"""

import torch

from .so2conv import Desc, _check_edges, edge_frame_rows, gate, unpack_weights
from .wigner import frame, wigner_d_blocks


def mix_rows(rows, w, desc: Desc):
    """Per-m mixing of edge-frame rows {(l, m): [E, C]} -> same keys.

    m = 0: v0 = W0 u0 with u0 = (rows[(l, 0)])_{l = 0..L};
    m >= 1: v+ = W1 u+ - W2 u-, v- = W2 u+ + W1 u-, u+- = (rows[(l, +-m)])_{l >= m}.
    """
    L, M, C = desc.lmax, desc.mmax, desc.c_out
    W0, pairs = unpack_weights(w, desc)
    out = {}
    u0 = torch.cat([rows[(l, 0)] for l in range(L + 1)], dim=-1)
    v0 = u0 @ W0.T
    for l in range(L + 1):
        out[(l, 0)] = v0[:, l * C:(l + 1) * C]
    for m in range(1, M + 1):
        W1, W2 = pairs[m - 1]
        up = torch.cat([rows[(l, m)] for l in range(m, L + 1)], dim=-1)
        um = torch.cat([rows[(l, -m)] for l in range(m, L + 1)], dim=-1)
        vp = up @ W1.T - um @ W2.T
        vm = up @ W2.T + um @ W1.T
        for l in range(m, L + 1):
            k = l - m
            out[(l, m)] = vp[:, k * C:(k + 1) * C]
            out[(l, -m)] = vm[:, k * C:(k + 1) * C]
    return out


def activation(h):
    """Every edge-frame row of a channel times sigmoid of its (0, 0) value."""
    sg = torch.sigmoid(h[(0, 0)])
    return {k: v * sg for k, v in h.items()}


def block_forward(x, src, dst, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2,
                  desc: Desc, n_nodes=None, roll=None):
    """x [N, S, C] -> out [N, S, C] (desc.c_in == desc.c_out == C)."""
    assert desc.c_in == desc.c_out, "the block keeps one channel count"
    L = desc.lmax
    n_nodes = x.shape[0] if n_nodes is None else n_nodes
    E = src.shape[0]
    out = x.new_zeros((n_nodes, desc.s, desc.c_out))
    if E == 0:
        return out + 0.0 * (w1.sum() + w2.sum() + w_rad1.sum() + w_rad2.sum() +
                            b_rad1.sum() + b_rad2.sum() + x.sum())
    d = _check_edges(edge_vec)
    R = frame(edge_vec / d[:, None])
    if roll is not None:
        c, s_ = torch.cos(roll), torch.sin(roll)
        o, z = torch.ones_like(c), torch.zeros_like(c)
        rz = torch.stack([torch.stack([c, -s_, z], -1),
                          torch.stack([s_, c, z], -1),
                          torch.stack([z, z, o], -1)], -2)
        R = rz @ R
    Ds = wigner_d_blocks(R, L)
    xs = x[src]
    full = [Ds[l] @ xs[:, l * l:(l + 1) ** 2, :] for l in range(L + 1)]
    a = {(l, m): full[l][:, l + m, :] for (l, m) in edge_frame_rows(desc)}
    g1 = gate(d, w_rad1, b_rad1, desc)
    h = {k: g1 * v for k, v in mix_rows(a, w1, desc).items()}
    hp = activation(h)
    g2 = gate(d, w_rad2, b_rad2, desc)
    yt = {k: g2 * v for k, v in mix_rows(hp, w2, desc).items()}
    zero = x.new_zeros((E, desc.c_out))
    ys = []
    for l in range(L + 1):
        t = torch.stack([yt.get((l, m), zero) for m in range(-l, l + 1)], 1)
        ys.append(Ds[l].transpose(-1, -2) @ t)
    return out.index_add(0, dst, torch.cat(ys, dim=1))


BLOCK_GRADS = ["grad_x", "grad_w1", "grad_w_rad1", "grad_b_rad1", "grad_w2", "grad_w_rad2",
               "grad_b_rad2", "grad_edge_vec"]


def block_backward(x, src, dst, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2,
                   desc: Desc, grad_out, n_nodes=None):
    """Exact first derivatives of <grad_out, block_forward(...)> (torch
    autograd in float64): a dict keyed by BLOCK_GRADS."""
    leaves = [t.detach().clone().requires_grad_(True)
              for t in (x, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2, edge_vec)]
    xl, w1l, wr1l, b1l, w2l, wr2l, b2l, rl = leaves
    out = block_forward(xl, src, dst, rl, w1l, wr1l, b1l, w2l, wr2l, b2l, desc, n_nodes)
    gs = torch.autograd.grad(out, leaves, grad_out, allow_unused=True)
    return {n: (g if g is not None else torch.zeros_like(t)).detach()
            for n, g, t in zip(BLOCK_GRADS, gs, leaves)}
