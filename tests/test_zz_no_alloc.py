"""so2conv_forward_noalloc: the forward for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run the convolution (inside a
stream capture they do not own, in a plugin whose host owns all device
memory, in a loop that must stay off the allocator).  This entry point runs
the forward on a fixed scratch array inside the library instead of a caller
workspace.  The test calls it through the C ABI twice in a row, on different
inputs, and checks each result against so2conv_forward and against the
float64 oracle, with the array's own status word read after each call; it
also checks that a problem too large for the array is refused before any
launch.  It lives in its own file so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from so_edge_convolution_b200 import binding as B
from so_edge_convolution_b200 import build, synth

from helpers import oracle_forward, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _tensors(p):
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    return (t(p.x), t(p.edge_index, torch.int64), t(p.edge_vec), t(p.w), t(p.w_rad),
            t(p.b_rad))


def test_forward_noalloc_matches_forward_on_two_calls():
    build.build()
    B.load()
    for seed in (0, 1):
        p = synth.make_problem("esen", seed=seed, n_atoms=200, max_nb=20, lmax=3, mmax=2,
                               c=32)
        desc = B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)
        args = _tensors(p)
        ref = B.forward(desc, *args)
        torch.cuda.synchronize()
        assert B.check(DEV) == 0
        got = B.forward_noalloc(desc, *args)
        assert B.noalloc_check(DEV) == 0
        err = ((got - ref).abs().max() / ref.abs().max()).item()
        assert err < 1e-4, (seed, err)
        assert rel_err(got, oracle_forward(p)) < 1e-4, seed


def test_forward_noalloc_refuses_a_problem_too_large():
    B.load()
    desc = B.make_desc(4, 2, 128, 128, 16, 6.0)
    assert B.workspace_size(desc, 20000, 1000000, B.WS_FORWARD) > (96 << 20)
    P = ctypes.c_void_p(0x1000)  # never dereferenced: refused before any launch
    code = B.load().so2conv_forward_noalloc(ctypes.byref(desc), 20000, 1000000, P, P, P,
                                            B.Params(0x1000, 0x1000, 0x1000), P, None)
    assert code == 3
