"""Pins for the oracle's edge frames and Wigner-D matrices (no GPU)."""

import math

import numpy as np
import pytest
import torch
from scipy.spatial.transform import Rotation

from oracle.sh import real_sh
from oracle.wigner import frame, wigner_d, wigner_d_blocks

P = torch.tensor([[0.0, 1.0, 0.0], [0.0, 0.0, 1.0], [1.0, 0.0, 0.0]],
                 dtype=torch.float64)  # (x, y, z) -> (y, z, x)


def _rots(n, seed):
    return torch.from_numpy(Rotation.random(n, random_state=seed).as_matrix())


def _dirs(n, seed):
    v = np.random.default_rng(seed).standard_normal((n, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    return torch.from_numpy(v)


def test_frame_maps_edge_to_z():
    special = torch.tensor([[0, 0, 1.0], [0, 0, -1.0], [1.0, 0, 0],
                            [0, 1.0, 0], [0.6, 0, -0.8], [1e-9, 0, -1.0]],
                           dtype=torch.float64)
    special = special / special.norm(dim=-1, keepdim=True)
    r = torch.cat([special, _dirs(200, 0)])
    R = frame(r)
    z = torch.tensor([0, 0, 1.0], dtype=torch.float64)
    assert torch.allclose(torch.einsum("eij,ej->ei", R, r),
                          z.expand_as(r), atol=1e-14)
    eye = torch.eye(3, dtype=torch.float64)
    assert torch.allclose(R @ R.transpose(-1, -2), eye.expand_as(R), atol=1e-14)
    assert torch.allclose(torch.linalg.det(R), torch.ones(len(r),
                          dtype=torch.float64), atol=1e-14)


@pytest.mark.parametrize("lmax", [2, 4, 6])
def test_orthogonal(lmax):
    D = wigner_d(_rots(20, 1), lmax)
    eye = torch.eye(D.shape[-1], dtype=torch.float64)
    assert (D @ D.transpose(-1, -2) - eye).abs().max() < 1e-13


def test_identity():
    D = wigner_d(torch.eye(3, dtype=torch.float64)[None], 6)[0]
    assert (D - torch.eye(49, dtype=torch.float64)).abs().max() < 1e-13


def test_defining_relation_on_fresh_directions():
    # Y(R n) = D(R) Y(n) on directions that were not used in the fit
    R = _rots(10, 2)
    n = _dirs(30, 3)
    D = wigner_d(R, 6)
    Yrn = real_sh(torch.einsum("rij,kj->rki", R, n), 6)
    DYn = torch.einsum("rst,kt->rks", D, real_sh(n, 6))
    assert (Yrn - DYn).abs().max() < 1e-12


def test_homomorphism():
    A, B = _rots(10, 4), _rots(10, 5)
    lhs = wigner_d(A @ B, 5)
    rhs = wigner_d(A, 5) @ wigner_d(B, 5)
    assert (lhs - rhs).abs().max() < 1e-12


def test_l1_block_is_permuted_rotation():
    R = _rots(10, 6)
    D1 = wigner_d_blocks(R, 1)[1]
    assert torch.allclose(D1, P @ R @ P.T, atol=1e-14)


def test_z_rotation_is_2x2_blocks():
    alpha = 0.7
    c, s = math.cos(alpha), math.sin(alpha)
    Rz = torch.tensor([[c, -s, 0], [s, c, 0], [0, 0, 1.0]],
                      dtype=torch.float64)[None]
    blocks = wigner_d_blocks(Rz, 4)
    for l, D in enumerate(blocks):
        D = D[0]
        for m in range(1, l + 1):
            cm, sm = math.cos(m * alpha), math.sin(m * alpha)
            assert abs(D[l + m, l + m] - cm) < 1e-13
            assert abs(D[l - m, l - m] - cm) < 1e-13
            assert abs(D[l + m, l - m] + sm) < 1e-13
            assert abs(D[l - m, l + m] - sm) < 1e-13
        assert abs(D[l, l] - 1.0) < 1e-13


def test_frame_sends_edge_harmonics_to_m0():
    r = _dirs(50, 7)
    D = wigner_d(frame(r), 6)
    Y = torch.einsum("est,et->es", D, real_sh(r, 6))
    for l in range(7):
        e = torch.zeros(2 * l + 1, dtype=torch.float64)
        e[l] = math.sqrt((2 * l + 1) / (4 * math.pi))
        assert (Y[:, l * l:(l + 1) ** 2] - e).abs().max() < 1e-12
