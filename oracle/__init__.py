"""Float64 CPU oracle for the SO(2) edge convolution.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
tables or constants with the CUDA library under
``so_edge_convolution_b200/csrc``; the two meet only through the seeded input
generators in ``so_edge_convolution_b200/synth.py``, which hold none of the
method's arithmetic.

What it computes follows the dataflow named in "TrimSO(2): Fast and
Memory-Efficient Training of Equivariant Interatomic Potentials" (Abstract):
rotate the source features into the edge frame, mix them per m with dense
matrices, recombine the +/-m pairs, gate with a radial term, rotate back and
reduce onto the destination node; backward and double backward are the exact
derivatives of that map (same Abstract: "higher-order differentiation").  The
page gives no formulas, so every convention below is a stated reading:

* real spherical harmonics, orthonormal, no Condon-Shortley phase, flat index
  l*l + l + m with m = -l..l, so the l = 1 block is (y, z, x);
* Wigner-D defined by Y(R n) = D(R) Y(n), found here by least squares over a
  fixed set of directions (no recursion, unlike the CUDA side);
* edge frame: any rotation R_e with R_e r_hat = z_hat; this oracle takes the
  minimal (Rodrigues) rotation, the CUDA side an azimuth/polar one;
* edge-frame rows with |m| > mmax are dropped;
* +/-m pair map: v+ = W1 u+ - W2 u-,  v- = W2 u+ + W1 u-;
* gate: g = W_rad^T phi(d) + b, Gaussian RBFs on linspace(0, cutoff, n_rbf)
  with width cutoff / (n_rbf - 1), applied per output channel after mixing;
* reduction: plain sum over incoming edges.

The message block (two such convolutions with an edge-frame activation
between them, the abstract's "recombination with activation") is in
``block.py``.

Parity status: every function here is pinned by tests/test_oracle_*.py against
closed forms, textbook tables, invariants and finite differences.
"""

from .so2conv import (  # noqa: F401
    Desc,
    block_shapes,
    n_weights,
    unpack_weights,
    rbf,
    gate,
    forward,
    forward_loop,
    backward,
    double_backward,
    edge_frame_rows,
)
from .block import (  # noqa: F401
    BLOCK_GRADS,
    activation,
    block_backward,
    block_forward,
    mix_rows,
)
from .sh import real_sh, legendre  # noqa: F401
from .wigner import frame, wigner_d, wigner_d_blocks  # noqa: F401
