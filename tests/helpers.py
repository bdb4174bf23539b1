"""Shared test helpers: problem -> tensors, oracle calls, error metrics."""

import dataclasses

import numpy as np
import torch

import oracle as O

F64 = torch.float64


def desc_of(p):
    return O.Desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)


def oracle_forward(p, edges=None):
    src, dst, vec = _edges(p, edges)
    return O.forward(torch.from_numpy(p.x), src, dst, vec, torch.from_numpy(p.w),
                     torch.from_numpy(p.w_rad), torch.from_numpy(p.b_rad), desc_of(p))


def oracle_backward(p, edges=None, grad_out=None):
    src, dst, vec = _edges(p, edges)
    G = torch.from_numpy(p.grad_out if grad_out is None else grad_out)
    return O.backward(torch.from_numpy(p.x), src, dst, vec, torch.from_numpy(p.w),
                      torch.from_numpy(p.w_rad), torch.from_numpy(p.b_rad), desc_of(p), G)


def oracle_double_backward(p, gg_x=None, gg_edge_vec=None, edges=None):
    src, dst, vec = _edges(p, edges)
    t = lambda a: None if a is None else torch.from_numpy(np.asarray(a, dtype=np.float64))  # noqa
    return O.double_backward(torch.from_numpy(p.x), src, dst, vec, torch.from_numpy(p.w),
                             torch.from_numpy(p.w_rad), torch.from_numpy(p.b_rad),
                             desc_of(p), torch.from_numpy(p.grad_out), gg_x=t(gg_x),
                             gg_edge_vec=t(gg_edge_vec))


def _edges(p, edges):
    ei, vec = p.edge_index, p.edge_vec
    if edges is not None:
        ei, vec = ei[:, edges], vec[edges]
    return (torch.from_numpy(ei[0].copy()), torch.from_numpy(ei[1].copy()),
            torch.from_numpy(vec.copy()))


def rel_err(gpu, ref):
    """max |gpu - ref| / max |ref| (the parity metric)."""
    gpu = gpu.detach().double().cpu() if torch.is_tensor(gpu) else torch.as_tensor(gpu, dtype=F64)
    ref = ref.detach().double().cpu() if torch.is_tensor(ref) else torch.as_tensor(ref, dtype=F64)
    scale = ref.abs().max().item()
    if scale == 0.0:
        return gpu.abs().max().item()
    return (gpu - ref).abs().max().item() / scale


def with_channels(p, c):
    """Embed a problem with C channels into one with c >= C channels (zeros)."""
    L, M, C = p.lmax, p.mmax, p.c_in
    S = (L + 1) ** 2
    x = np.zeros((p.n_nodes, S, c))
    x[:, :, :C] = p.x
    blocks, off = [], 0
    from so_edge_convolution_b200.synth import weight_block_shapes
    for (r, k), (r2, k2) in zip(weight_block_shapes(L, M, C, C), weight_block_shapes(L, M, c, c)):
        B = p.w[off:off + r * k].reshape(r // C, C, k // C, C)
        off += r * k
        Bn = np.zeros((r2 // c, c, k2 // c, c))
        Bn[:, :C, :, :C] = B
        blocks.append(Bn.reshape(-1))
    w_rad = np.zeros((p.n_rbf, c))
    w_rad[:, :C] = p.w_rad
    b = np.zeros(c)
    b[:C] = p.b_rad
    G = np.zeros((p.n_nodes, S, c))
    G[:, :, :C] = p.grad_out
    return dataclasses.replace(p, c_in=c, c_out=c, x=x, w=np.concatenate(blocks),
                               w_rad=w_rad, b_rad=b, grad_out=G)
