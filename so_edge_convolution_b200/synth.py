"""Seeded synthetic inputs for the SO(2) edge convolution.

This module only draws inputs: atom positions, neighbour lists, edge vectors,
node features, weights and cotangents.  It holds none of the convolution's
arithmetic and is the one module that both the float64 oracle's tests and the
CUDA path's tests and benchmark use, so that both see identical values.

Workloads (the pages measure on eSEN / UMA / EquiformerV3 training sets that
are not available here; these synthetic graphs stand in for them):

* ``tiny``  64 atoms uniform in an open 10 A cube, each destination takes its
  16 nearest sources within 5 A; lmax = mmax = 2, C = 16, 8 RBFs, fp32.
* ``esen``  2,000 atoms in a periodic cube at 0.1 atoms/A^3 (side 27.14 A),
  30 nearest within 6 A (E = 60,000); lmax 4, mmax 2, C 128, 16 RBFs, fp32.
* ``force`` the ``esen`` graph and shapes, with the energy cotangent
  (grad_out = 1 on the l = 0 rows) and a force target F_ref.
* ``uma``   5,000 atoms at the same density, 30 neighbours (E = 150,000);
  lmax 6, mmax 2, C 128, bf16 features and weights.
* ``large`` 20,000 atoms, 50 neighbours (E = 1,000,000); lmax 4, mmax 2,
  C 128, bf16 features.

Draw order from one ``numpy.random.default_rng(seed)``: positions, x, the
weight blocks in packed order, W_rad, b_rad, grad_out, F_ref.  Every array is
drawn in float64; bf16 configurations round x (and for ``uma`` the weights)
to bf16 once, and both sides take those rounded values.
"""

import dataclasses

import numpy as np
from scipy.spatial import cKDTree

CONFIGS = {
    "tiny": dict(n_atoms=64, box=10.0, periodic=False, cutoff=5.0, max_nb=16,
                 lmax=2, mmax=2, c=16, n_rbf=8, rbf_cutoff=5.0,
                 x_bf16=False, w_bf16=False),
    "esen": dict(n_atoms=2000, density=0.1, periodic=True, cutoff=6.0,
                 max_nb=30, lmax=4, mmax=2, c=128, n_rbf=16, rbf_cutoff=6.0,
                 x_bf16=False, w_bf16=False),
    "force": dict(n_atoms=2000, density=0.1, periodic=True, cutoff=6.0,
                  max_nb=30, lmax=4, mmax=2, c=128, n_rbf=16, rbf_cutoff=6.0,
                  x_bf16=False, w_bf16=False, energy_cotangent=True),
    "uma": dict(n_atoms=5000, density=0.1, periodic=True, cutoff=6.0,
                max_nb=30, lmax=6, mmax=2, c=128, n_rbf=16, rbf_cutoff=6.0,
                x_bf16=True, w_bf16=True),
    "large": dict(n_atoms=20000, density=0.1, periodic=True, cutoff=6.0,
                  max_nb=50, lmax=4, mmax=2, c=128, n_rbf=16, rbf_cutoff=6.0,
                  x_bf16=True, w_bf16=False),
}


@dataclasses.dataclass
class Problem:
    name: str
    lmax: int
    mmax: int
    c_in: int
    c_out: int
    n_rbf: int
    rbf_cutoff: float
    pos: np.ndarray          # [N, 3] float64
    x: np.ndarray            # [N, S, c_in] float64 (bf16-exact when x_bf16)
    edge_index: np.ndarray   # [2, E] int64, row 0 = src, row 1 = dst
    edge_vec: np.ndarray     # [E, 3] float64, pos[src] - pos[dst] + shift
    w: np.ndarray            # packed weight blocks, float64
    w_rad: np.ndarray        # [n_rbf, c_out]
    b_rad: np.ndarray        # [c_out]
    grad_out: np.ndarray     # [N, S, c_out]
    f_ref: np.ndarray        # [N, 3]
    x_bf16: bool
    w_bf16: bool

    @property
    def n_nodes(self):
        return self.x.shape[0]

    @property
    def n_edges(self):
        return self.edge_index.shape[1]

    @property
    def s(self):
        return (self.lmax + 1) ** 2


def weight_block_shapes(lmax, mmax, c_in, c_out):
    """Packed weight layout: W0 then (W1_m, W2_m) for m = 1..mmax."""
    shapes = [((lmax + 1) * c_out, (lmax + 1) * c_in)]
    for m in range(1, mmax + 1):
        k = lmax + 1 - m
        shapes += [(k * c_out, k * c_in), (k * c_out, k * c_in)]
    return shapes


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (through torch) and widen back."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def neighbour_graph(pos, box, periodic, cutoff, max_nb):
    """Each destination keeps its max_nb nearest sources within cutoff.

    Returns (edge_index [2, E], edge_vec [E, 3]) in destination-major order,
    nearest first.  Periodic boxes use the minimum image.
    """
    n = pos.shape[0]
    tree = cKDTree(pos, boxsize=box if periodic else None)
    k = min(max_nb + 1, n)
    dist, idx = tree.query(pos, k=k, distance_upper_bound=cutoff)
    src_l, dst_l = [], []
    for i in range(n):
        keep = [(d, j) for d, j in zip(dist[i], idx[i])
                if j < n and j != i and d < cutoff]
        keep.sort(key=lambda t: (t[0], t[1]))
        for d, j in keep[:max_nb]:
            src_l.append(j)
            dst_l.append(i)
    src = np.asarray(src_l, dtype=np.int64)
    dst = np.asarray(dst_l, dtype=np.int64)
    vec = pos[src] - pos[dst]
    if periodic:
        vec -= box * np.round(vec / box)
    return np.stack([src, dst]), vec


def make_problem(name: str, seed: int = 0, n_atoms=None, max_nb=None,
                 lmax=None, mmax=None, c=None) -> Problem:
    """Draw one synthetic workload; overrides shrink it for parity tests."""
    cfg = dict(CONFIGS[name])
    if n_atoms is not None:
        cfg["n_atoms"] = n_atoms
    if max_nb is not None:
        cfg["max_nb"] = max_nb
    if lmax is not None:
        cfg["lmax"] = lmax
    if mmax is not None:
        cfg["mmax"] = mmax
    if c is not None:
        cfg["c"] = c
    rng = np.random.default_rng(seed)
    n = cfg["n_atoms"]
    if cfg["periodic"]:
        box = (n / cfg["density"]) ** (1.0 / 3.0)
    else:
        box = cfg["box"]
    pos = rng.uniform(0.0, box, size=(n, 3))
    L, M, C = cfg["lmax"], cfg["mmax"], cfg["c"]
    S = (L + 1) ** 2
    x = rng.standard_normal((n, S, C))
    blocks = []
    for r, k in weight_block_shapes(L, M, C, C):
        blocks.append(rng.standard_normal((r, k)).reshape(-1) / np.sqrt(k))
    w = np.concatenate(blocks)
    nr = cfg["n_rbf"]
    w_rad = rng.standard_normal((nr, C)) / np.sqrt(nr)
    b_rad = rng.standard_normal(C) / np.sqrt(nr)
    if cfg.get("energy_cotangent"):
        grad_out = np.zeros((n, S, C))
        grad_out[:, 0, :] = 1.0
        rng.standard_normal((n, S, C))  # keep the draw order fixed
    else:
        grad_out = rng.standard_normal((n, S, C))
    f_ref = rng.standard_normal((n, 3))
    if cfg["x_bf16"]:
        x = round_bf16(x)
    if cfg["w_bf16"]:
        w = round_bf16(w)
    ei, vec = neighbour_graph(pos, box, cfg["periodic"], cfg["cutoff"],
                              cfg["max_nb"])
    return Problem(name=name, lmax=L, mmax=M, c_in=C, c_out=C, n_rbf=nr,
                   rbf_cutoff=cfg["rbf_cutoff"], pos=pos, x=x, edge_index=ei,
                   edge_vec=vec, w=w, w_rad=w_rad, b_rad=b_rad,
                   grad_out=grad_out, f_ref=f_ref, x_bf16=cfg["x_bf16"],
                   w_bf16=cfg["w_bf16"])


def shuffled(p: Problem, seed: int = 1) -> Problem:
    """The same problem with its edges in a seeded random order."""
    perm = np.random.default_rng(seed).permutation(p.n_edges)
    return dataclasses.replace(p, edge_index=p.edge_index[:, perm].copy(),
                               edge_vec=p.edge_vec[perm].copy())


def random_graph(n_nodes, n_edges, lmax, mmax, c_in, c_out, n_rbf=8,
                 cutoff=5.0, seed=0, min_sep=0.8):
    """Small random multigraph for gradient checks.

    Edge vectors are drawn with length in [min_sep, cutoff) so that no frame
    is undefined; src and dst are independent uniform node ids.
    """
    rng = np.random.default_rng(seed)
    S = (lmax + 1) ** 2
    x = rng.standard_normal((n_nodes, S, c_in))
    src = rng.integers(0, n_nodes, n_edges)
    dst = rng.integers(0, n_nodes, n_edges)
    dirs = rng.standard_normal((n_edges, 3))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    lens = rng.uniform(min_sep, cutoff, n_edges)
    vec = dirs * lens[:, None]
    blocks = []
    for r, k in weight_block_shapes(lmax, mmax, c_in, c_out):
        blocks.append(rng.standard_normal((r, k)).reshape(-1) / np.sqrt(k))
    w = np.concatenate(blocks)
    w_rad = rng.standard_normal((n_rbf, c_out)) / np.sqrt(n_rbf)
    b_rad = rng.standard_normal(c_out) / np.sqrt(n_rbf)
    grad_out = rng.standard_normal((n_nodes, S, c_out))
    return Problem(name="random", lmax=lmax, mmax=mmax, c_in=c_in,
                   c_out=c_out, n_rbf=n_rbf, rbf_cutoff=cutoff,
                   pos=np.zeros((n_nodes, 3)), x=x,
                   edge_index=np.stack([src, dst]).astype(np.int64),
                   edge_vec=vec, w=w, w_rad=w_rad, b_rad=b_rad,
                   grad_out=grad_out, f_ref=rng.standard_normal((n_nodes, 3)),
                   x_bf16=False, w_bf16=False)
