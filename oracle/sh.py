"""Real spherical harmonics in float64 (oracle; test infrastructure only).

Convention (a reading: the pages print no basis, see "TrimSO(2): Fast and
Memory-Efficient Training of Equivariant Interatomic Potentials", Abstract,
which only names the rotations):

    Y_{l,0}  = N_l0 P_l(z)
    Y_{l,m}  = sqrt(2) N_lm P_l^{(m)}(z) Re((x + i y)^m)      m > 0
    Y_{l,-m} = sqrt(2) N_lm P_l^{(m)}(z) Im((x + i y)^m)      m > 0
    N_lm     = sqrt((2l+1)/(4 pi) * (l-m)! / (l+m)!)

for a unit vector n = (x, y, z).  P_l^{(m)} is the m-th derivative of the
Legendre polynomial, so P_l^{(m)}(z) Re((x+iy)^m) = P_l^m(cos t) cos(m phi)
without the Condon-Shortley phase.  Every expression is a polynomial in
(x, y, z), so torch autograd differentiates it to any order.
"""

import math

import numpy as np
import torch
from numpy.polynomial import legendre as npleg
from numpy.polynomial import polynomial as nppoly


def legendre(l: int, z: torch.Tensor) -> torch.Tensor:
    """P_l(z) by numpy's Legendre-to-power-series conversion and Horner."""
    coef = npleg.leg2poly([0.0] * l + [1.0])
    return _horner(coef, z)


def _horner(coef, z):
    out = torch.zeros_like(z)
    for c in coef[::-1]:
        out = out * z + float(c)
    return out


def _legendre_deriv_coef(l: int, m: int):
    coef = npleg.leg2poly([0.0] * l + [1.0])
    for _ in range(m):
        coef = nppoly.polyder(coef)
    return coef


def real_sh(n: torch.Tensor, lmax: int) -> torch.Tensor:
    """Y(n) for all l <= lmax: [..., 3] -> [..., (lmax+1)^2], flat l*l+l+m."""
    x, y, z = n[..., 0], n[..., 1], n[..., 2]
    cols = []
    # (x + i y)^m as (re, im) pairs, m = 0..lmax
    re = [torch.ones_like(x)]
    im = [torch.zeros_like(x)]
    for m in range(1, lmax + 1):
        re.append(re[-1] * x - im[-1] * y)
        im.append(re[-2] * y + im[-1] * x)
    for l in range(lmax + 1):
        row = [None] * (2 * l + 1)
        for m in range(0, l + 1):
            nlm = math.sqrt((2 * l + 1) / (4 * math.pi)
                            * math.factorial(l - m) / math.factorial(l + m))
            p = _horner(_legendre_deriv_coef(l, m), z)
            if m == 0:
                row[l] = nlm * p
            else:
                row[l + m] = math.sqrt(2.0) * nlm * p * re[m]
                row[l - m] = math.sqrt(2.0) * nlm * p * im[m]
        cols.extend(row)
    return torch.stack(cols, dim=-1)


def fixed_directions(count: int = 96, seed: int = 12345) -> torch.Tensor:
    """A fixed, well spread set of unit vectors used to fit Wigner-D."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((count, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    return torch.from_numpy(v)
