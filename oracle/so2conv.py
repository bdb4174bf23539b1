"""The SO(2) edge convolution, written out plainly in float64 (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring for the conventions).

Per edge e = (s -> d) with edge vector r_e, the map is
("TrimSO(2): Fast and Memory-Efficient Training of Equivariant Interatomic
Potentials", Abstract: rotation on gather, dense per-m mixing, recombination,
inverse rotation on reduction):

    R_e r_hat_e = z_hat                     edge frame
    a      = trunc(D(R_e) x[s])             rotate into the frame, keep |m|<=mmax
    v0     = W0 u0                          m = 0, u0 = (a[l,0,:])_l
    v+     = W1_m u+ - W2_m u-              m > 0, u+- = (a[l,+-m,:])_{l>=m}
    v-     = W2_m u+ + W1_m u-
    y~     = g(|r_e|) * v                   per output channel gate
    out[d] += D(R_e)^T y~                   rotate back and sum

Backward and double backward are the exact derivatives of this map, taken by
torch autograd in float64 (pinned by central finite differences in the tests).
"""

import dataclasses

import torch

from .wigner import frame, wigner_d, wigner_d_blocks


@dataclasses.dataclass(frozen=True)
class Desc:
    lmax: int
    mmax: int
    c_in: int
    c_out: int
    n_rbf: int
    cutoff: float

    @property
    def s(self):
        return (self.lmax + 1) ** 2


def edge_frame_rows(desc: Desc):
    """(l, m) rows kept in the edge frame: |m| <= min(l, mmax), l-major."""
    return [(l, m) for l in range(desc.lmax + 1)
            for m in range(-min(l, desc.mmax), min(l, desc.mmax) + 1)]


def block_shapes(desc: Desc):
    """Shapes of the packed weight blocks: W0, then (W1_m, W2_m), m=1..mmax.

    Rows are (l' - m) * c_out + c', columns (l - m) * c_in + c.
    """
    L = desc.lmax
    shapes = [((L + 1) * desc.c_out, (L + 1) * desc.c_in)]
    for m in range(1, desc.mmax + 1):
        k = L + 1 - m
        shapes.append((k * desc.c_out, k * desc.c_in))
        shapes.append((k * desc.c_out, k * desc.c_in))
    return shapes


def n_weights(desc: Desc) -> int:
    return sum(r * c for r, c in block_shapes(desc))


def unpack_weights(w: torch.Tensor, desc: Desc):
    """Flat packed vector -> (W0, [(W1_1, W2_1), (W1_2, W2_2), ...])."""
    blocks = []
    off = 0
    for r, c in block_shapes(desc):
        blocks.append(w[off:off + r * c].reshape(r, c))
        off += r * c
    assert off == w.numel()
    pairs = [(blocks[1 + 2 * i], blocks[2 + 2 * i]) for i in range(desc.mmax)]
    return blocks[0], pairs


def rbf(d: torch.Tensor, desc: Desc) -> torch.Tensor:
    """Gaussian radial basis: centres linspace(0, cutoff, n_rbf), width
    cutoff / (n_rbf - 1), no envelope and no normalisation."""
    mu = torch.linspace(0.0, desc.cutoff, desc.n_rbf, dtype=d.dtype)
    sigma = desc.cutoff / (desc.n_rbf - 1)
    return torch.exp(-((d[:, None] - mu[None, :]) ** 2) / (2.0 * sigma * sigma))


def gate(d, w_rad, b_rad, desc: Desc):
    """Radial gate g = W_rad^T phi(d) + b: [E] -> [E, c_out]."""
    return rbf(d, desc) @ w_rad + b_rad[None, :]


def _check_edges(edge_vec):
    d = torch.linalg.norm(edge_vec, dim=-1)
    if edge_vec.shape[0] and bool((d == 0).any()):
        raise ValueError("zero-length edge: its frame is undefined")
    return d


def forward(x, src, dst, edge_vec, w, w_rad, b_rad, desc: Desc, n_nodes=None,
            roll=None):
    """Batched float64 forward.  x [N, S, c_in] -> out [N, S, c_out].

    ``roll`` (optional, [E] radians) turns each edge frame about z_hat; the
    result must not depend on it (tests use this to check roll invariance).
    """
    L, M = desc.lmax, desc.mmax
    n_nodes = x.shape[0] if n_nodes is None else n_nodes
    E = src.shape[0]
    out = x.new_zeros((n_nodes, desc.s, desc.c_out))
    if E == 0:
        return out + 0.0 * (w.sum() + w_rad.sum() + b_rad.sum() + x.sum())
    d = _check_edges(edge_vec)
    rhat = edge_vec / d[:, None]
    R = frame(rhat)
    if roll is not None:
        c, s_ = torch.cos(roll), torch.sin(roll)
        o, z = torch.ones_like(c), torch.zeros_like(c)
        rz = torch.stack([torch.stack([c, -s_, z], -1),
                          torch.stack([s_, c, z], -1),
                          torch.stack([z, z, o], -1)], -2)
        R = rz @ R
    Ds = wigner_d_blocks(R, L)
    g = gate(d, w_rad, b_rad, desc)
    xs = x[src]
    a = [Ds[l] @ xs[:, l * l:(l + 1) ** 2, :] for l in range(L + 1)]
    W0, pairs = unpack_weights(w, desc)
    co = desc.c_out
    rows = {}  # (l', m) -> [E, c_out] gated edge-frame output
    u0 = torch.cat([a[l][:, l, :] for l in range(L + 1)], dim=-1)
    v0 = u0 @ W0.T
    for lp in range(L + 1):
        rows[(lp, 0)] = g * v0[:, lp * co:(lp + 1) * co]
    for m in range(1, M + 1):
        W1, W2 = pairs[m - 1]
        up = torch.cat([a[l][:, l + m, :] for l in range(m, L + 1)], dim=-1)
        um = torch.cat([a[l][:, l - m, :] for l in range(m, L + 1)], dim=-1)
        vp = up @ W1.T - um @ W2.T
        vm = up @ W2.T + um @ W1.T
        for lp in range(m, L + 1):
            k = lp - m
            rows[(lp, m)] = g * vp[:, k * co:(k + 1) * co]
            rows[(lp, -m)] = g * vm[:, k * co:(k + 1) * co]
    zero = x.new_zeros((E, co))
    ys = []
    for l in range(L + 1):
        yt = torch.stack([rows.get((l, m), zero) for m in range(-l, l + 1)], 1)
        ys.append(Ds[l].transpose(-1, -2) @ yt)
    y = torch.cat(ys, dim=1)
    return out.index_add(0, dst, y)


def forward_loop(x, src, dst, edge_vec, w, w_rad, b_rad, desc: Desc,
                 n_nodes=None):
    """Second formulation, one edge at a time with a dense edge-frame matrix.

    For each edge the full mixing map M (S*c_out x S*c_in, zero outside the
    kept rows) is assembled entry by entry from the weight blocks, and
    out[d] += (D^T (x) I) diag(g) M (D (x) I) vec(x[s]).  Meant for tiny
    graphs only; it checks the batched forward by brute force.
    """
    L, M = desc.lmax, desc.mmax
    S, ci, co = desc.s, desc.c_in, desc.c_out
    n_nodes = x.shape[0] if n_nodes is None else n_nodes
    W0, pairs = unpack_weights(w, desc)

    def idx(l, m):
        return l * l + l + m

    Mfull = x.new_zeros((S * co, S * ci))
    for lp in range(L + 1):
        for l in range(L + 1):
            for cp in range(co):
                for c in range(ci):
                    Mfull[idx(lp, 0) * co + cp, idx(l, 0) * ci + c] = \
                        W0[lp * co + cp, l * ci + c]
    for m in range(1, M + 1):
        W1, W2 = pairs[m - 1]
        for lp in range(m, L + 1):
            for l in range(m, L + 1):
                for cp in range(co):
                    for c in range(ci):
                        r1 = W1[(lp - m) * co + cp, (l - m) * ci + c]
                        r2 = W2[(lp - m) * co + cp, (l - m) * ci + c]
                        op, om = idx(lp, m) * co + cp, idx(lp, -m) * co + cp
                        ip, im = idx(l, m) * ci + c, idx(l, -m) * ci + c
                        Mfull[op, ip] = r1
                        Mfull[op, im] = -r2
                        Mfull[om, ip] = r2
                        Mfull[om, im] = r1
    out = x.new_zeros((n_nodes, S, co))
    for e in range(src.shape[0]):
        r = edge_vec[e]
        dist = torch.linalg.norm(r)
        D = wigner_d(frame((r / dist)[None]), L)[0]
        g = gate(dist[None], w_rad, b_rad, desc)[0]
        Din = torch.kron(D, torch.eye(ci, dtype=x.dtype))
        Dout = torch.kron(D, torch.eye(co, dtype=x.dtype))
        gvec = g.repeat(S)
        y = Dout.T @ (gvec * (Mfull @ (Din @ x[src[e]].reshape(-1))))
        out[dst[e]] += y.reshape(S, co)
    return out


def _leaves(*ts):
    return [t.detach().clone().requires_grad_(True) for t in ts]


def backward(x, src, dst, edge_vec, w, w_rad, b_rad, desc: Desc, grad_out,
             n_nodes=None):
    """Exact first derivatives of <grad_out, forward(...)>.

    Returns a dict with grad_x, grad_w, grad_w_rad, grad_b_rad, grad_edge_vec.
    """
    xl, wl, wrl, bl, rl = _leaves(x, w, w_rad, b_rad, edge_vec)
    out = forward(xl, src, dst, rl, wl, wrl, bl, desc, n_nodes)
    gs = torch.autograd.grad(out, [xl, wl, wrl, bl, rl], grad_out,
                             allow_unused=True)
    names = ["grad_x", "grad_w", "grad_w_rad", "grad_b_rad", "grad_edge_vec"]
    ref = [xl, wl, wrl, bl, rl]
    return {n: (g if g is not None else torch.zeros_like(t)).detach()
            for n, g, t in zip(names, gs, ref)}


def double_backward(x, src, dst, edge_vec, w, w_rad, b_rad, desc: Desc,
                    grad_out, gg_x=None, gg_edge_vec=None, n_nodes=None):
    """Derivatives of Q = <gg_x, grad_x> + <gg_edge_vec, grad_edge_vec>.

    grad_x and grad_edge_vec are the first-order gradients of
    <grad_out, forward(...)>.  Returns d_x, d_w, d_w_rad, d_b_rad,
    d_grad_out and d_edge_vec (all exact, float64).
    """
    xl, wl, wrl, bl, rl, gl = _leaves(x, w, w_rad, b_rad, edge_vec, grad_out)
    out = forward(xl, src, dst, rl, wl, wrl, bl, desc, n_nodes)
    gx, gw, gwr, gb, gr = torch.autograd.grad(
        out, [xl, wl, wrl, bl, rl], gl, create_graph=True, allow_unused=True)
    q = out.new_zeros(())
    if gg_x is not None and gx is not None:
        q = q + (gg_x * gx).sum()
    if gg_edge_vec is not None and gr is not None:
        q = q + (gg_edge_vec * gr).sum()
    ref = [xl, wl, wrl, bl, gl, rl]
    if not q.requires_grad:
        return {n: torch.zeros_like(t).detach() for n, t in zip(
            ["d_x", "d_w", "d_w_rad", "d_b_rad", "d_grad_out", "d_edge_vec"],
            ref)}
    ds = torch.autograd.grad(q, ref, allow_unused=True)
    names = ["d_x", "d_w", "d_w_rad", "d_b_rad", "d_grad_out", "d_edge_vec"]
    return {n: (g if g is not None else torch.zeros_like(t)).detach()
            for n, g, t in zip(names, ds, ref)}


def mixing_flops_per_edge(desc: Desc) -> int:
    """Multiply-add count x2 of one pass of the per-m mixing for one edge."""
    k0 = (desc.lmax + 1)
    f = 2 * (k0 * desc.c_out) * (k0 * desc.c_in)
    for m in range(1, desc.mmax + 1):
        k = desc.lmax + 1 - m
        f += 4 * 2 * (k * desc.c_out) * (k * desc.c_in)
    return f



