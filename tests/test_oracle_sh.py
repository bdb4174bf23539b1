"""Pins for the oracle's real spherical harmonics (no GPU).

The basis is a reading (the pages print none): real, orthonormal, no
Condon-Shortley phase, m = -l..l, l = 1 ordered (y, z, x).  These tests tie it
to textbook closed forms, quadrature orthonormality, the addition theorem and
parity, none of which reuse the oracle's own formula.
"""

import math

import numpy as np
import pytest
import torch
from scipy.special import eval_legendre

from oracle.sh import real_sh

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _rand_dirs(n, seed):
    v = np.random.default_rng(seed).standard_normal((n, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    return torch.from_numpy(v)


def test_textbook_l_le_2():
    n = _rand_dirs(50, 0)
    x, y, z = n[:, 0], n[:, 1], n[:, 2]
    Y = real_sh(n, 2)
    pi = math.pi
    expect = [
        torch.full_like(x, 0.5 * math.sqrt(1 / pi)),
        math.sqrt(3 / (4 * pi)) * y,
        math.sqrt(3 / (4 * pi)) * z,
        math.sqrt(3 / (4 * pi)) * x,
        0.5 * math.sqrt(15 / pi) * x * y,
        0.5 * math.sqrt(15 / pi) * y * z,
        0.25 * math.sqrt(5 / pi) * (3 * z * z - 1),
        0.5 * math.sqrt(15 / pi) * x * z,
        0.25 * math.sqrt(15 / pi) * (x * x - y * y),
    ]
    for i, e in enumerate(expect):
        assert torch.allclose(Y[:, i], e, atol=1e-14, rtol=0), i


def test_l3_closed_forms():
    n = _rand_dirs(40, 1)
    x, y, z = n[:, 0], n[:, 1], n[:, 2]
    Y = real_sh(n, 3)
    pi = math.pi
    # l = 3: m = 0 and m = +-3 (textbook real forms, no phase)
    e0 = 0.25 * math.sqrt(7 / pi) * z * (5 * z * z - 3)
    e3 = 0.25 * math.sqrt(35 / (2 * pi)) * x * (x * x - 3 * y * y)
    em3 = 0.25 * math.sqrt(35 / (2 * pi)) * y * (3 * x * x - y * y)
    assert torch.allclose(Y[:, 12], e0, atol=1e-14)
    assert torch.allclose(Y[:, 15], e3, atol=1e-14)
    assert torch.allclose(Y[:, 9], em3, atol=1e-14)


@pytest.mark.parametrize("lmax", [4, 6])
def test_orthonormal_by_quadrature(lmax):
    # Gauss-Legendre in z times a uniform azimuth grid integrates
    # polynomials of degree <= 2*lmax on the sphere exactly.
    nz, nphi = lmax + 2, 2 * lmax + 3
    zq, wq = np.polynomial.legendre.leggauss(nz)
    phi = 2 * np.pi * np.arange(nphi) / nphi
    Z, P = np.meshgrid(zq, phi, indexing="ij")
    W = np.repeat(wq[:, None], nphi, 1) * (2 * np.pi / nphi)
    rho = np.sqrt(1 - Z * Z)
    pts = np.stack([rho * np.cos(P), rho * np.sin(P), Z], -1).reshape(-1, 3)
    Y = real_sh(torch.from_numpy(pts), lmax).numpy()
    G = (Y * W.reshape(-1, 1)).T @ Y
    assert np.abs(G - np.eye(G.shape[0])).max() < 1e-12


@pytest.mark.parametrize("l", [0, 1, 2, 3, 4, 5, 6])
def test_addition_theorem(l):
    a, b = _rand_dirs(30, 2), _rand_dirs(30, 3)
    Ya = real_sh(a, l)[:, l * l:]
    Yb = real_sh(b, l)[:, l * l:]
    lhs = (Ya * Yb).sum(-1).numpy()
    cos = (a * b).sum(-1).numpy()
    rhs = (2 * l + 1) / (4 * np.pi) * eval_legendre(l, cos)
    assert np.abs(lhs - rhs).max() < 1e-13


def test_parity():
    n = _rand_dirs(20, 4)
    Y, Yn = real_sh(n, 6), real_sh(-n, 6)
    for l in range(7):
        sl = slice(l * l, (l + 1) ** 2)
        assert torch.allclose(Yn[:, sl], (-1) ** l * Y[:, sl], atol=1e-13)
