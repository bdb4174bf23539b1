"""Edge frames and real Wigner-D matrices in float64 (oracle; test only).

D^l(R) is fixed by its defining relation Y_l(R n) = D^l(R) Y_l(n) for every
unit vector n ("rotation on gather" / "inverse rotation on reduction" in
"TrimSO(2): Fast and Memory-Efficient Training of Equivariant Interatomic
Potentials", Abstract, rotate features by this matrix and by its transpose).
Here it is solved exactly (up to rounding) by least squares over a fixed set
of directions N:  D^l(R) = Y_l(R N) pinv(Y_l(N)).  No recursion is used, so
this shares nothing with the CUDA generator.
"""

import torch

from .sh import fixed_directions, real_sh

_PINV_CACHE = {}


def _pinv_table(lmax: int):
    key = lmax
    if key not in _PINV_CACHE:
        dirs = fixed_directions()
        y = real_sh(dirs, lmax)  # [K, S]
        tabs = []
        for l in range(lmax + 1):
            yl = y[:, l * l:(l + 1) * (l + 1)].T  # [2l+1, K]
            tabs.append(torch.linalg.pinv(yl))  # [K, 2l+1]
        _PINV_CACHE[key] = (dirs, tabs)
    return _PINV_CACHE[key]


def wigner_d_blocks(R: torch.Tensor, lmax: int):
    """List over l of D^l(R): [..., 2l+1, 2l+1]; R is [..., 3, 3]."""
    dirs, tabs = _pinv_table(lmax)
    rn = torch.einsum("...ij,kj->...ki", R, dirs)  # R applied to each n_k
    y = real_sh(rn, lmax)  # [..., K, S]
    # l = 0 is the trivial representation: exactly 1 (Y_00 is constant)
    blocks = [torch.ones(R.shape[:-2] + (1, 1), dtype=R.dtype) + 0.0 * R[..., :1, :1]]
    for l in range(1, lmax + 1):
        yl = y[..., l * l:(l + 1) * (l + 1)].transpose(-1, -2)  # [..., 2l+1, K]
        blocks.append(yl @ tabs[l])
    return blocks


def wigner_d(R: torch.Tensor, lmax: int) -> torch.Tensor:
    """Block-diagonal D(R): [..., S, S] with S = (lmax+1)^2."""
    blocks = wigner_d_blocks(R, lmax)
    s = (lmax + 1) ** 2
    out = R.new_zeros(R.shape[:-2] + (s, s))
    for l, b in enumerate(blocks):
        out[..., l * l:(l + 1) ** 2, l * l:(l + 1) ** 2] = b
    return out


def _skew(v):
    z = torch.zeros_like(v[..., 0])
    return torch.stack([
        torch.stack([z, -v[..., 2], v[..., 1]], -1),
        torch.stack([v[..., 2], z, -v[..., 0]], -1),
        torch.stack([-v[..., 1], v[..., 0], z], -1),
    ], -2)


def frame(rhat: torch.Tensor) -> torch.Tensor:
    """Rotation R with R rhat = z_hat, for unit rhat [..., 3] -> [..., 3, 3].

    Minimal (Rodrigues) rotation onto +z when rhat_z >= 0.  When rhat_z < 0
    it first takes rhat onto -z the same way, then turns by pi about x; this
    keeps 1 + cos(angle) away from zero.  The roll about z that this choice
    fixes has no effect on the convolution's output.
    """
    eye = torch.eye(3, dtype=rhat.dtype).expand(rhat.shape[:-1] + (3, 3))
    up = rhat[..., 2] >= 0
    target_z = torch.where(up, torch.ones_like(rhat[..., 2]),
                           -torch.ones_like(rhat[..., 2]))
    tgt = torch.stack([torch.zeros_like(target_z), torch.zeros_like(target_z),
                       target_z], -1)
    v = torch.cross(rhat, tgt, dim=-1)
    c = (rhat * tgt).sum(-1)
    k = _skew(v)
    R = eye + k + (k @ k) / (1.0 + c)[..., None, None]
    flip = torch.diag(torch.tensor([1.0, -1.0, -1.0], dtype=rhat.dtype))
    R = torch.where(up[..., None, None], R, flip @ R)
    return R
