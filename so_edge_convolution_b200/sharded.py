"""One graph over several GPUs: destination-partitioned edges.

Each rank owns a contiguous range of nodes and the edges whose destination
it owns, so the convolution's reduction onto nodes stays local.  The one
exchange is around it:

* forward: every rank's node features are all-gathered into the full node
  array (the gather side may read any node), the rank's edges are convolved,
  and the output rows of its own nodes are complete;
* backward: the rank's edges give partial gradients; grad_x (whose rows are
  the edges' sources, owned anywhere) is summed over ranks and scattered to
  the owners, the weight gradients are summed over ranks, and the edge-vector
  gradients stay with the rank's edges.

Local node arrays have `per` rows (the last rank's tail zero-padded) so that
every collective moves equal blocks.  `op` is the module that runs the
convolution on one device: the C-ABI binding by default.  The collectives
are torch.distributed's (NCCL over NVLink on GPUs).
"""

import torch
import torch.distributed as dist


def node_range(n_nodes, rank, world):
    """(n0, n1, per): the rank's nodes [n0, n1) and the padded rows per rank."""
    per = -(-n_nodes // world)
    n0 = min(rank * per, n_nodes)
    n1 = min(n0 + per, n_nodes)
    return n0, n1, per


class ShardedGraph:
    """The rank's share of a graph given in full (edge_index [2, E], edge_vec
    [E, 3], any device): its node range and its edges, in global edge order."""

    def __init__(self, edge_index, edge_vec, n_nodes, rank=None, world=None, group=None):
        self.group = group
        self.rank = dist.get_rank(group) if rank is None else rank
        self.world = dist.get_world_size(group) if world is None else world
        self.n_nodes = n_nodes
        self.n0, self.n1, self.per = node_range(n_nodes, self.rank, self.world)
        dst = edge_index[1]
        keep = (dst >= self.n0) & (dst < self.n1)
        self.edge_ids = torch.nonzero(keep).flatten()
        self.edge_index = edge_index[:, self.edge_ids].contiguous()
        self.edge_vec = edge_vec[self.edge_ids].contiguous()

    @property
    def n_pad(self):
        return self.per * self.world

    def local_rows(self, full):
        """This rank's `per` rows of a full [N, ...] node array (zero-padded)."""
        out = full.new_zeros((self.per,) + tuple(full.shape[1:]))
        out[: self.n1 - self.n0] = full[self.n0:self.n1]
        return out

    def gather_nodes(self, local):
        """All ranks' [per, ...] rows -> the full [n_pad, ...] node array."""
        local = local.contiguous()
        full = local.new_empty((self.n_pad,) + tuple(local.shape[1:]))
        if dist.get_backend(self.group) == "gloo":
            dist.all_gather(list(full.chunk(self.world)), local, group=self.group)
        else:
            dist.all_gather_into_tensor(full, local, group=self.group)
        return full

    def reduce_nodes(self, full):
        """Sum a full [n_pad, ...] node array over ranks; this rank's rows."""
        full = full.contiguous()
        if dist.get_backend(self.group) == "gloo":  # no reduce-scatter on gloo
            dist.all_reduce(full, group=self.group)
            return full[self.rank * self.per:(self.rank + 1) * self.per].clone()
        out = full.new_empty((self.per,) + tuple(full.shape[1:]))
        dist.reduce_scatter_tensor(out, full, group=self.group)
        return out

    def reduce_all(self, t):
        dist.all_reduce(t, group=self.group)
        return t


def _op(op):
    if op is None:
        from so_edge_convolution_b200 import binding as op_default
        return op_default
    return op


def forward(sg, desc, x_local, w, w_rad, b_rad, op=None):
    """Output rows [per, S, C_out] of this rank's nodes."""
    op = _op(op)
    x_full = sg.gather_nodes(x_local)
    out_full = op.forward(desc, x_full, sg.edge_index, sg.edge_vec, w, w_rad, b_rad)
    return out_full[sg.rank * sg.per:(sg.rank + 1) * sg.per]


def backward(sg, desc, x_local, w, w_rad, b_rad, grad_out_local, op=None):
    """Gradients: grad_x rows of this rank's nodes [per, S, C_in], the summed
    weight gradients, and grad_edge_vec of this rank's edges (global edge ids
    in sg.edge_ids)."""
    op = _op(op)
    x_full = sg.gather_nodes(x_local)
    g_full = grad_out_local.new_zeros((sg.n_pad,) + tuple(grad_out_local.shape[1:]))
    g_full[sg.rank * sg.per:(sg.rank + 1) * sg.per] = grad_out_local
    g = op.backward(desc, x_full, sg.edge_index, sg.edge_vec, w, w_rad, b_rad, g_full)
    res = {"grad_x": sg.reduce_nodes(g["grad_x"]), "grad_edge_vec": g["grad_edge_vec"]}
    for k in ("grad_w", "grad_w_rad", "grad_b_rad"):
        res[k] = sg.reduce_all(g[k].contiguous())
    return res
