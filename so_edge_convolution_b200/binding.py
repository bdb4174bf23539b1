"""Thin ctypes binding of libso2conv (include/so2conv.h) for torch tensors.

Argument marshalling only: every step of the convolution runs in the
library's CUDA kernels.  Torch supplies device memory (inputs, outputs and
the workspace) and the current stream.  If the shared library is missing or
does not load, every call raises -- there is no fallback path.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libso2conv.so")

SO2_F32, SO2_BF16 = 0, 1
WS_FORWARD, WS_BACKWARD, WS_DOUBLE_BACKWARD = 0, 1, 2
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace",
          4: "cuda", 5: "index", 6: "timeout", 7: "degenerate edge"}


class Desc(ctypes.Structure):
    _fields_ = [("lmax", ctypes.c_int32), ("mmax", ctypes.c_int32),
                ("c_in", ctypes.c_int32), ("c_out", ctypes.c_int32),
                ("n_rbf", ctypes.c_int32), ("rbf_cutoff", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class Params(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("w_rad", ctypes.c_void_p),
                ("b_rad", ctypes.c_void_p)]


class So2Error(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


_lib = None


def load():
    """Load libso2conv.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with "
            "`python -m so_edge_convolution_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    pd = ctypes.POINTER(Desc)
    lib.so2conv_workspace_size.argtypes = [pd, i64, i64, ctypes.c_int]
    lib.so2conv_workspace_size.restype = sz
    lib.so2conv_num_weights.argtypes = [pd]
    lib.so2conv_num_weights.restype = i64
    lib.so2conv_forward.argtypes = [pd, i64, i64, vp, vp, vp, Params, vp, vp, sz, vp]
    lib.so2conv_forward.restype = ctypes.c_int
    lib.so2conv_backward.argtypes = [pd, i64, i64, vp, vp, vp, Params, vp, vp, vp, vp,
                                     vp, vp, vp, sz, vp]
    lib.so2conv_backward.restype = ctypes.c_int
    lib.so2conv_double_backward.argtypes = [pd, i64, i64, vp, vp, vp, Params, vp, vp, vp,
                                            vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.so2conv_double_backward.restype = ctypes.c_int
    lib.so2conv_check.argtypes = [vp, vp]
    lib.so2conv_check.restype = ctypes.c_int
    lib.so2conv_status_string.argtypes = [ctypes.c_int]
    lib.so2conv_status_string.restype = ctypes.c_char_p
    lib.so2conv_edge_frames.argtypes = [ctypes.c_int32, i64, vp, vp, vp, vp]
    lib.so2conv_edge_frames.restype = ctypes.c_int
    lib.so2conv_forward_noalloc.argtypes = [pd, i64, i64, vp, vp, vp, Params, vp, vp]
    lib.so2conv_forward_noalloc.restype = ctypes.c_int
    lib.so2conv_block_workspace_size.argtypes = [pd, i64, i64, ctypes.c_int]
    lib.so2conv_block_workspace_size.restype = sz
    lib.so2conv_block_forward.argtypes = [pd, i64, i64, vp, vp, vp, Params, Params, vp, vp, sz, vp]
    lib.so2conv_block_forward.restype = ctypes.c_int
    lib.so2conv_block_backward.argtypes = [pd, i64, i64, vp, vp, vp, Params, Params, vp,
                                           vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.so2conv_block_backward.restype = ctypes.c_int
    lib.so2conv_noalloc_check.argtypes = [vp]
    lib.so2conv_noalloc_check.restype = ctypes.c_int
    lib.so2conv_launch_count.argtypes = []
    lib.so2conv_launch_count.restype = ctypes.c_longlong
    lib.so2conv_wait_selftest.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64,
                                          ctypes.c_void_p]
    lib.so2conv_wait_selftest.restype = ctypes.c_int
    lib.so2conv_set_max_chunk_edges.argtypes = [ctypes.c_int64]
    lib.so2conv_set_max_chunk_edges.restype = ctypes.c_int
    lib.so2conv_max_chunk_edges.argtypes = []
    lib.so2conv_max_chunk_edges.restype = ctypes.c_int64
    lib.so2conv_profile_enable.argtypes = [ctypes.c_int]
    lib.so2conv_profile_enable.restype = None
    lib.so2conv_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_double)]
    lib.so2conv_profile_read.restype = ctypes.c_int
    _lib = lib
    return lib


def make_desc(lmax, mmax, c_in, c_out, n_rbf, rbf_cutoff, dtype=SO2_F32):
    return Desc(lmax, mmax, c_in, c_out, n_rbf, float(rbf_cutoff), dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("so2conv tensors must be contiguous (row-major)")
    return ctypes.c_void_p(t.data_ptr())


def _c(t):
    return None if t is None else t.contiguous()


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_call(code, where):
    if code != 0:
        raise So2Error(code, where)


class Workspace:
    """A reusable device workspace (grown on demand, 256-byte aligned)."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = None

    def get(self, nbytes):
        if self.buf is None or self.buf.numel() < nbytes + 256:
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8,
                                   device=self.device)
        base = self.buf.data_ptr()
        off = (-base) % 256
        return ctypes.c_void_p(base + off), nbytes


_WS = {}


def workspace(device):
    key = torch.device(device)
    if key not in _WS:
        _WS[key] = Workspace(key)
    return _WS[key]


def num_weights(desc):
    return int(load().so2conv_num_weights(ctypes.byref(desc)))


def workspace_size(desc, n_nodes, n_edges, which):
    return int(load().so2conv_workspace_size(ctypes.byref(desc), n_nodes, n_edges, which))


def _wsarg(desc, n_nodes, n_edges, which, device, ws):
    need = workspace_size(desc, n_nodes, n_edges, which)
    if need == 0:
        raise So2Error(2, "workspace_size")
    w = ws or workspace(device)
    return w.get(need)


def forward(desc, x, edge_index, edge_vec, w, w_rad, b_rad, out=None, ws=None):
    lib = load()
    x, edge_index, edge_vec, w, w_rad, b_rad = map(_c, (x, edge_index, edge_vec, w, w_rad, b_rad))
    N, E = x.shape[0], edge_index.shape[1]
    if out is None:
        out = torch.empty((N, (desc.lmax + 1) ** 2, desc.c_out), dtype=torch.float32,
                          device=x.device)
    p, nb = _wsarg(desc, N, E, WS_FORWARD, x.device, ws)
    code = lib.so2conv_forward(ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index),
                               _ptr(edge_vec), Params(_ptr(w).value, _ptr(w_rad).value, _ptr(b_rad).value),
                               _ptr(out), p, nb, _stream(x.device))
    _check_call(code, "so2conv_forward")
    return out


def _outputs(names, need, shapes, out, f32):
    """The output tensors: caller-given ones (checked) or new ones."""
    res = {}
    for n in names:
        if n not in need:
            res[n] = None
        elif out is not None and out.get(n) is not None:
            t = out[n]
            if (tuple(t.shape) != tuple(shapes[n]) or t.dtype != torch.float32
                    or t.device != f32["device"] or not t.is_contiguous()):
                raise ValueError(f"out[{n!r}] must be a contiguous float32 tensor of shape "
                                 f"{tuple(shapes[n])} on {f32['device']}")
            res[n] = t
        else:
            res[n] = torch.empty(shapes[n], **f32)
    return res


def backward(desc, x, edge_index, edge_vec, w, w_rad, b_rad, grad_out, need=None,
             ws=None, out=None):
    """Returns a dict of gradients; `need` limits which ones are computed and
    `out` (a dict) may give preallocated tensors for some of them."""
    lib = load()
    x, edge_index, edge_vec, w, w_rad, b_rad, grad_out = map(
        _c, (x, edge_index, edge_vec, w, w_rad, b_rad, grad_out))
    N, E = x.shape[0], edge_index.shape[1]
    names = ["grad_x", "grad_w", "grad_w_rad", "grad_b_rad", "grad_edge_vec"]
    need = set(names if need is None else need)
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    S = (desc.lmax + 1) ** 2
    shapes = {"grad_x": (N, S, desc.c_in), "grad_w": (num_weights(desc),),
              "grad_w_rad": (desc.n_rbf, desc.c_out), "grad_b_rad": (desc.c_out,),
              "grad_edge_vec": (E, 3)}
    outs = _outputs(names, need, shapes, out, f32)
    p, nb = _wsarg(desc, N, E, WS_BACKWARD, dev, ws)
    code = lib.so2conv_backward(ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index),
                                _ptr(edge_vec), Params(w.data_ptr(), w_rad.data_ptr(),
                                                       b_rad.data_ptr()),
                                _ptr(grad_out), *[_ptr(outs[n]) for n in names], p, nb,
                                _stream(dev))
    _check_call(code, "so2conv_backward")
    return {n: t for n, t in outs.items() if t is not None}


def double_backward(desc, x, edge_index, edge_vec, w, w_rad, b_rad, grad_out, gg_x=None,
                    gg_edge_vec=None, need=None, ws=None, out=None):
    lib = load()
    x, edge_index, edge_vec, w, w_rad, b_rad, grad_out, gg_x, gg_edge_vec = map(
        _c, (x, edge_index, edge_vec, w, w_rad, b_rad, grad_out, gg_x, gg_edge_vec))
    N, E = x.shape[0], edge_index.shape[1]
    names = ["d_x", "d_w", "d_w_rad", "d_b_rad", "d_grad_out", "d_edge_vec"]
    need = set(names if need is None else need)
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    S = (desc.lmax + 1) ** 2
    shapes = {"d_x": (N, S, desc.c_in), "d_w": (num_weights(desc),),
              "d_w_rad": (desc.n_rbf, desc.c_out), "d_b_rad": (desc.c_out,),
              "d_grad_out": (N, S, desc.c_out), "d_edge_vec": (E, 3)}
    outs = _outputs(names, need, shapes, out, f32)
    p, nb = _wsarg(desc, N, E, WS_DOUBLE_BACKWARD, dev, ws)
    code = lib.so2conv_double_backward(
        ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index), _ptr(edge_vec),
        Params(w.data_ptr(), w_rad.data_ptr(), b_rad.data_ptr()), _ptr(grad_out),
        _ptr(gg_x), _ptr(gg_edge_vec), *[_ptr(outs[n]) for n in names], p, nb,
        _stream(dev))
    _check_call(code, "so2conv_double_backward")
    return {n: t for n, t in outs.items() if t is not None}


def check(device, ws=None):
    """Synchronise and return the device status of the last call (0 = ok)."""
    w = ws or workspace(device)
    if w.buf is None:
        return 0
    base = w.buf.data_ptr()
    return int(load().so2conv_check(ctypes.c_void_p(base + (-base) % 256),
                                    _stream(device)))


def edge_frames(lmax, edge_vec):
    """Frames R [E, 3, 3] and full Wigner-D blocks [E, Dsz] as the library
    computes them."""
    E = edge_vec.shape[0]
    dsz = sum((2 * l + 1) ** 2 for l in range(lmax + 1))
    R = torch.empty((E, 9), dtype=torch.float32, device=edge_vec.device)
    D = torch.empty((E, dsz), dtype=torch.float32, device=edge_vec.device)
    code = load().so2conv_edge_frames(lmax, E, _ptr(edge_vec), _ptr(R), _ptr(D),
                                      _stream(edge_vec.device))
    _check_call(code, "so2conv_edge_frames")
    return R.view(E, 3, 3), D


def wait_selftest(device, limit_us=1000):
    """so2conv_wait_selftest, then so2conv_check: returns the recorded status
    (SO2_ERR_TIMEOUT = 6 when the bounded wait gave up as it should)."""
    lib = load()
    w = workspace(device)
    p, nb = w.get(256)
    _check_call(lib.so2conv_wait_selftest(p, nb, int(limit_us), _stream(device)),
                "so2conv_wait_selftest")
    return int(lib.so2conv_check(p, _stream(device)))


def set_max_chunk_edges(n):
    """so2conv_set_max_chunk_edges: edges per chunk of per-edge intermediates
    (0 restores the default); returns the value now in force."""
    lib = load()
    _check_call(lib.so2conv_set_max_chunk_edges(int(n)), "so2conv_set_max_chunk_edges")
    return int(lib.so2conv_max_chunk_edges())


def launch_count():
    """Kernels launched by the library so far in this process."""
    return int(load().so2conv_launch_count())


def profile_enable(on=True, all_kinds=False):
    """Record CUDA events around the tensor-core launches (and, with
    all_kinds, around every group of CUDA-core launches too)."""
    load().so2conv_profile_enable((2 if all_kinds else 1) if on else 0)


PROFILE_KINDS = {0: "mixing (x W^T)", 1: "mixing transposed (g W)", 2: "weight gradient",
                 3: "rotation on gather", 4: "edge preparation", 5: "edge gradient terms",
                 6: "radial sums", 7: "weight packing and node scatter"}
TENSOR_KINDS = (0, 1, 2)


def profile_read():
    """{kind: (ranges, total_ms)} of the recorded launches (kinds 0-2: one
    range per tcgen05 launch; 3-7: groups of CUDA-core launches)."""
    lib = load()
    res = {}
    for k in PROFILE_KINDS:
        n, ms = ctypes.c_int(0), ctypes.c_double(0.0)
        _check_call(lib.so2conv_profile_read(k, ctypes.byref(n), ctypes.byref(ms)),
                    "so2conv_profile_read")
        res[k] = (n.value, ms.value)
    return res


def forward_noalloc(desc, x, edge_index, edge_vec, w, w_rad, b_rad, out=None):
    """so2conv_forward_noalloc: the forward on the library's own scratch array
    (no workspace argument, nothing allocated by the library)."""
    lib = load()
    x, edge_index, edge_vec, w, w_rad, b_rad = map(_c, (x, edge_index, edge_vec, w, w_rad, b_rad))
    N, E = x.shape[0], edge_index.shape[1]
    if out is None:
        out = torch.empty((N, (desc.lmax + 1) ** 2, desc.c_out), dtype=torch.float32,
                          device=x.device)
    code = lib.so2conv_forward_noalloc(ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index),
                                       _ptr(edge_vec), Params(_ptr(w).value, _ptr(w_rad).value,
                                                              _ptr(b_rad).value),
                                       _ptr(out), _stream(x.device))
    _check_call(code, "so2conv_forward_noalloc")
    return out


def noalloc_check(device):
    """Synchronise and return the device status of the last no-alloc forward
    in the current context (0 = ok)."""
    return int(load().so2conv_noalloc_check(_stream(device)))


# ---------------------------------------------------------------------------
# Message block: two convolutions with the edge-frame activation between them
# ---------------------------------------------------------------------------
BLOCK_GRADS = ["grad_x", "grad_w1", "grad_w_rad1", "grad_b_rad1", "grad_w2", "grad_w_rad2",
               "grad_b_rad2", "grad_edge_vec"]


def block_workspace_size(desc, n_nodes, n_edges, which):
    return int(load().so2conv_block_workspace_size(ctypes.byref(desc), n_nodes, n_edges, which))


def _block_ws(desc, n_nodes, n_edges, which, device, ws):
    need = block_workspace_size(desc, n_nodes, n_edges, which)
    if need == 0:
        raise So2Error(2, "block_workspace_size")
    return (ws or workspace(device)).get(need)


def _params(w, w_rad, b_rad):
    return Params(_ptr(w).value, _ptr(w_rad).value, _ptr(b_rad).value)


def block_forward(desc, x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2,
                  out=None, ws=None):
    """so2conv_block_forward: out [N, S, C] of the two-convolution block."""
    lib = load()
    x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2 = map(
        _c, (x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2))
    N, E = x.shape[0], edge_index.shape[1]
    if out is None:
        out = torch.empty((N, (desc.lmax + 1) ** 2, desc.c_out), dtype=torch.float32,
                          device=x.device)
    p, nb = _block_ws(desc, N, E, 0, x.device, ws)
    code = lib.so2conv_block_forward(ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index),
                                     _ptr(edge_vec), _params(w1, w_rad1, b_rad1),
                                     _params(w2, w_rad2, b_rad2), _ptr(out), p, nb,
                                     _stream(x.device))
    _check_call(code, "so2conv_block_forward")
    return out


def block_backward(desc, x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2,
                   grad_out, need=None, ws=None, out=None):
    """so2conv_block_backward: a dict keyed by BLOCK_GRADS (those in `need`)."""
    lib = load()
    x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2, grad_out = map(
        _c, (x, edge_index, edge_vec, w1, w_rad1, b_rad1, w2, w_rad2, b_rad2, grad_out))
    N, E = x.shape[0], edge_index.shape[1]
    need = set(BLOCK_GRADS if need is None else need)
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    S = (desc.lmax + 1) ** 2
    nw = num_weights(desc)
    shapes = {"grad_x": (N, S, desc.c_in), "grad_w1": (nw,), "grad_w2": (nw,),
              "grad_w_rad1": (desc.n_rbf, desc.c_out), "grad_w_rad2": (desc.n_rbf, desc.c_out),
              "grad_b_rad1": (desc.c_out,), "grad_b_rad2": (desc.c_out,),
              "grad_edge_vec": (E, 3)}
    outs = _outputs(BLOCK_GRADS, need, shapes, out, f32)
    p, nb = _block_ws(desc, N, E, 1, dev, ws)
    code = lib.so2conv_block_backward(ctypes.byref(desc), N, E, _ptr(x), _ptr(edge_index),
                                      _ptr(edge_vec), _params(w1, w_rad1, b_rad1),
                                      _params(w2, w_rad2, b_rad2), _ptr(grad_out),
                                      *[_ptr(outs[n]) for n in BLOCK_GRADS], p, nb, _stream(dev))
    _check_call(code, "so2conv_block_backward")
    return {n: t for n, t in outs.items() if t is not None}
