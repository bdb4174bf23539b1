"""The C ABI without a GPU: the library loads, exports every declared entry
point, sizes workspaces and rejects bad arguments before touching a device."""

import ctypes
import os
import re

import pytest

import oracle as O
from so_edge_convolution_b200 import binding as B
from so_edge_convolution_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.load()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^[a-z_0-9 *]+?\b(so2conv_\w+)\s*\(", txt, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "so2conv_forward" in names and "so2conv_double_backward" in names
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("L,M,ci,co", [(2, 2, 16, 16), (4, 2, 128, 128), (6, 2, 128, 128),
                                       (3, 0, 32, 48), (5, 5, 16, 32)])
def test_num_weights_matches_layout(lib, L, M, ci, co):
    d = B.make_desc(L, M, ci, co, 8, 5.0)
    assert B.num_weights(d) == O.n_weights(O.Desc(L, M, ci, co, 8, 5.0))


def test_workspace_sizes(lib):
    d = B.make_desc(4, 2, 128, 128, 16, 6.0)
    f = B.workspace_size(d, 2000, 60000, B.WS_FORWARD)
    b = B.workspace_size(d, 2000, 60000, B.WS_BACKWARD)
    assert 0 < f < b
    assert B.workspace_size(d, 0, 0, B.WS_FORWARD) > 0
    bad = B.make_desc(7, 2, 128, 128, 16, 6.0)
    assert B.workspace_size(bad, 10, 10, B.WS_FORWARD) == 0


def test_chunk_size_knob(lib):
    d = B.make_desc(4, 2, 128, 128, 16, 6.0, B.SO2_F32)
    assert B.set_max_chunk_edges(0) == 65536
    big = B.workspace_size(d, 2000, 200000, B.WS_BACKWARD)
    try:
        assert B.set_max_chunk_edges(1000) == 1024
        small = B.workspace_size(d, 2000, 200000, B.WS_BACKWARD)
        assert 0 < small < big
        assert lib.so2conv_set_max_chunk_edges(-1) == 1  # SO2_ERR_INVALID_ARG
        assert lib.so2conv_set_max_chunk_edges(1 << 23) == 1
        assert lib.so2conv_max_chunk_edges() == 1024
    finally:
        B.set_max_chunk_edges(0)
    assert B.workspace_size(d, 2000, 200000, B.WS_BACKWARD) == big


def _fwd(lib, desc, N=4, E=3, x=1, ei=1, ev=1, w=1, ws=1, nbytes=None):
    # (never dereferenced) f = 2: a pointer that is not 16-byte aligned
    P = lambda f: ctypes.c_void_p({0: 0, 1: 0x1000, 2: 0x1008}[f])  # noqa: E731
    prm = B.Params(0x1000 if w else 0, 0x1000, 0x1000)
    nb = nbytes if nbytes is not None else (1 << 40)
    return lib.so2conv_forward(ctypes.byref(desc), N, E, P(x), P(ei), P(ev), prm,
                               ctypes.c_void_p(0x2000), ctypes.c_void_p(0x100000 if ws else 0),
                               nb, None)


def test_argument_errors_are_reported_before_any_launch(lib):
    good = B.make_desc(2, 2, 16, 16, 8, 5.0)
    assert _fwd(lib, B.make_desc(7, 2, 16, 16, 8, 5.0)) == 2       # lmax > 6
    assert _fwd(lib, B.make_desc(2, 3, 16, 16, 8, 5.0)) == 2       # mmax > lmax
    assert _fwd(lib, B.make_desc(2, 2, 24, 16, 8, 5.0)) == 2       # c_in % 16
    assert _fwd(lib, B.make_desc(2, 2, 16, 16, 1, 5.0)) == 2       # n_rbf < 2
    assert _fwd(lib, good, x=0) == 1
    assert _fwd(lib, good, x=2) == 1                                 # x not 16-byte aligned
    assert _fwd(lib, good, ei=0) == 1
    assert _fwd(lib, good, w=0) == 1
    assert _fwd(lib, good, ws=0) == 3
    assert _fwd(lib, good, nbytes=16) == 3
    assert _fwd(lib, good, N=-1) == 1
    assert lib.so2conv_forward(None, 1, 1, None, None, None, B.Params(0, 0, 0), None, None, 0,
                               None) == 1


def test_status_strings(lib):
    for code in range(8):
        s = lib.so2conv_status_string(code)
        assert s and len(s) > 1


def test_block_argument_errors_are_reported_before_any_launch(lib):
    # (never dereferenced) the block's checks run before any CUDA call
    P = ctypes.c_void_p(0x1000)
    good = B.Params(0x1000, 0x1000, 0x1000)

    def fwd(desc, p2=good, nbytes=1 << 40, x=P):
        return lib.so2conv_block_forward(ctypes.byref(desc), 4, 3, x, P, P, good, p2,
                                         ctypes.c_void_p(0x2000), ctypes.c_void_p(0x100000),
                                         nbytes, None)
    d = B.make_desc(2, 2, 16, 16, 8, 5.0)
    assert fwd(B.make_desc(2, 2, 16, 32, 8, 5.0)) == 2        # the block keeps one C
    assert fwd(B.make_desc(7, 2, 16, 16, 8, 5.0)) == 2        # lmax > 6
    assert fwd(d, p2=B.Params(0, 0x1000, 0x1000)) == 1        # second conv's weights
    assert fwd(d, x=None) == 1
    assert fwd(d, nbytes=B.block_workspace_size(d, 4, 3, 0) - 1) == 3
    # the block's workspace holds the single convolution's and more
    assert B.block_workspace_size(d, 4, 3, 0) > B.workspace_size(d, 4, 3, B.WS_FORWARD)
    assert B.block_workspace_size(d, 4, 3, 1) > B.workspace_size(d, 4, 3, B.WS_BACKWARD)
    assert B.block_workspace_size(d, 4, 3, 2) == 0
