"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Tolerances (max |gpu - ref| / max |ref| per output tensor): 1e-4 for the f32
path (bf16 hi/lo split products, f32 accumulation), 2e-2 for bf16 inputs.
The reduction set and the per-edge output order are checked exactly.
"""

import dataclasses
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from so_edge_convolution_b200 import binding as B
from so_edge_convolution_b200 import synth

from helpers import (oracle_backward, oracle_forward, rel_err, with_channels)

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
TOL = {False: 1e-4, True: 2e-2}
DEV = "cuda:0"


def _desc(p):
    bf = p.x_bf16
    return B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff,
                       B.SO2_BF16 if bf else B.SO2_F32)


def _dev(p):
    dt = torch.bfloat16 if p.x_bf16 else torch.float32
    t = lambda a, d=torch.float32: torch.as_tensor(np.asarray(a)).to(d).to(DEV)  # noqa: E731
    return dict(x=t(p.x, dt), edge_index=t(p.edge_index, torch.int64),
                edge_vec=t(p.edge_vec), w=t(p.w, dt), w_rad=t(p.w_rad), b_rad=t(p.b_rad),
                grad_out=t(p.grad_out))


def _gpu_forward(p):
    d = _dev(p)
    out = B.forward(_desc(p), d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                    d["b_rad"])
    assert B.check(DEV) == 0
    return out


def _gpu_backward(p, need=None):
    d = _dev(p)
    g = B.backward(_desc(p), d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                   d["b_rad"], d["grad_out"], need=need)
    assert B.check(DEV) == 0
    return g


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from so_edge_convolution_b200 import build
    build.build()
    B.load()
    torch.cuda.init()


# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lmax", [2, 4, 6])
def test_frames_and_wigner_d(lmax):
    # lmax <= 4 runs the register-carried recursion, lmax 6 the one that reads
    # each previous block back from shared memory
    rng = np.random.default_rng(0)
    v = rng.standard_normal((500, 3)) * 3
    v[:6] = [[0, 0, 2], [0, 0, -2], [1, 0, 0], [0, 1e-7, -1], [1e-6, 0, 1], [0, -3, 0]]
    ev = torch.tensor(v, dtype=torch.float32, device=DEV)
    R, D = B.edge_frames(lmax, ev)
    R64 = R.double().cpu()
    rh = torch.tensor(v / np.linalg.norm(v, axis=1, keepdims=True))
    z = torch.einsum("eij,ej->ei", R64, rh)
    assert (z - torch.tensor([0, 0, 1.0], dtype=torch.float64)).abs().max() < 2e-6
    eye = torch.eye(3, dtype=torch.float64)
    assert (R64 @ R64.transpose(1, 2) - eye).abs().max() < 2e-6
    ref = O.wigner_d_blocks(R64, lmax)
    off = 0
    for l in range(lmax + 1):
        n = (2 * l + 1) ** 2
        got = D[:, off:off + n].double().cpu().view(-1, 2 * l + 1, 2 * l + 1)
        assert (got - ref[l]).abs().max() < 5e-6, l
        off += n


def _hand_cases():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: c["name"])
def test_hand_derived_cases(case):
    L, M = case["lmax"], case["mmax"]
    base = synth.Problem(name="hand", lmax=L, mmax=M, c_in=1, c_out=1, n_rbf=case["n_rbf"],
                         rbf_cutoff=case["cutoff"], pos=np.zeros((2, 3)),
                         x=np.asarray(case["x"], float)[..., None],
                         edge_index=np.asarray(case["edge_index"], np.int64),
                         edge_vec=np.asarray(case["edge_vec"], float),
                         w=np.asarray(case["w"], float), w_rad=np.asarray(case["w_rad"], float),
                         b_rad=np.asarray(case["b_rad"], float),
                         grad_out=np.zeros((2, (L + 1) ** 2, 1)), f_ref=np.zeros((2, 3)),
                         x_bf16=False, w_bf16=False)
    p = with_channels(base, 16)
    out = _gpu_forward(p).cpu().double()
    expect = torch.tensor(case["out"], dtype=torch.float64)
    # f32 gate (exp) and products: ~1e-7 relative
    assert (out[..., 0] - expect).abs().max() <= 1e-6 * max(1.0, expect.abs().max().item())
    assert out[..., 1:].abs().max() == 0


def _small(L=3, M=2, C=32, n=300, nb=30, seed=0, bf16=False):
    p = synth.make_problem("esen", seed=seed, n_atoms=n, max_nb=nb, lmax=L, mmax=M, c=C)
    if bf16:
        p = dataclasses.replace(p, x=synth.round_bf16(p.x), w=synth.round_bf16(p.w),
                                x_bf16=True, w_bf16=True)
    return p


@pytest.fixture(autouse=True)
def _small_chunks_for_chunked_cases(request):
    # cases named *_chunks run with 2,048-edge chunks (1,024 in the double
    # backward), so that small graphs cross several chunk boundaries
    params = getattr(getattr(request.node, "callspec", None), "params", {})
    chunked = "chunks" in str(params.get("name", ""))
    if chunked:
        B.set_max_chunk_edges(2048)
    yield
    if chunked:
        B.set_max_chunk_edges(0)


CASES = [
    ("tiny", lambda: synth.make_problem("tiny")),
    ("L3M2C32_chunks", lambda: _small(L=3, M=2, C=32, n=300, nb=30)),  # 9,000 edges, 5 chunks
    ("L4M2C128_bf16_chunks", lambda: _small(L=4, M=2, C=128, n=180, nb=25, seed=6, bf16=True)),
    ("L4M2C128_ragged", lambda: _small(L=4, M=2, C=128, n=150, nb=23, seed=1)),
    ("L2M0C16", lambda: _small(L=2, M=0, C=16, n=100, nb=11, seed=2)),
    ("L6M2C48_bf16", lambda: _small(L=6, M=2, C=48, n=120, nb=17, seed=3, bf16=True)),
    ("L4M2C128_bf16", lambda: _small(L=4, M=2, C=128, n=100, nb=25, seed=4, bf16=True)),
    ("L5M5C16", lambda: _small(L=5, M=5, C=16, n=60, nb=9, seed=5)),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_forward_parity(name, make):
    p = make()
    out = _gpu_forward(p)
    ref = oracle_forward(p)
    assert rel_err(out, ref) < TOL[p.x_bf16], name


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_backward_parity(name, make):
    p = make()
    g = _gpu_backward(p)
    ref = oracle_backward(p)
    for k in ["grad_x", "grad_w", "grad_w_rad", "grad_b_rad", "grad_edge_vec"]:
        err = rel_err(g[k], ref[k])
        assert err < TOL[p.x_bf16], (name, k, err)


def test_backward_partial_outputs():
    p = _small(L=3, M=2, C=32, n=80, nb=12, seed=6)
    full = _gpu_backward(p)
    for need in (["grad_x"], ["grad_w"], ["grad_edge_vec"], ["grad_w_rad", "grad_b_rad"]):
        part = _gpu_backward(p, need=need)
        assert set(part) == set(need)
        for k in need:
            # node sums are reduced with atomics: the order may differ per run
            assert rel_err(part[k], full[k]) < 1e-6, k


def _integer_problem(n=200, nb=20, seed=7):
    p = synth.make_problem("esen", seed=seed, n_atoms=n, max_nb=nb, lmax=2, mmax=2, c=16)
    x = np.zeros_like(p.x)
    x[:, 0, :] = np.arange(n)[:, None]
    blocks = [np.zeros(r * k) for r, k in synth.weight_block_shapes(2, 2, 16, 16)]
    W0 = np.zeros((48, 48))
    W0[:16, :16] = np.eye(16)
    blocks[0] = W0.reshape(-1)
    G = np.zeros_like(p.grad_out)
    G[:, 0, :] = np.arange(n)[:, None]
    return dataclasses.replace(p, x=x, w=np.concatenate(blocks), w_rad=np.zeros_like(p.w_rad),
                               b_rad=np.ones_like(p.b_rad), grad_out=G)


@pytest.mark.parametrize("shuffle", [False, True])
def test_reduction_set_is_exact(shuffle):
    p = _integer_problem()
    if shuffle:
        p = synth.shuffled(p, seed=3)
    src, dst = p.edge_index
    out = _gpu_forward(p).cpu().double().numpy()
    sum_src = np.bincount(dst, weights=src, minlength=p.n_nodes)
    assert np.array_equal(out[:, 0, 0], sum_src)
    assert np.all(out[:, 1:, :] == 0)
    gx = _gpu_backward(p, need=["grad_x"])["grad_x"].cpu().double().numpy()
    sum_dst = np.bincount(src, weights=dst, minlength=p.n_nodes)
    assert np.array_equal(gx[:, 0, 0], sum_dst)
    # degrees
    q = dataclasses.replace(p, x=np.where(p.x != 0, 1.0, 1.0) * (np.arange(p.s) == 0)[None, :, None])
    deg = _gpu_forward(q).cpu().double().numpy()[:, 0, 0]
    assert np.array_equal(deg, np.bincount(dst, minlength=p.n_nodes).astype(float))


def test_edge_order_is_kept():
    p = _small(L=3, M=2, C=32, n=120, nb=15, seed=8)
    q = synth.shuffled(p, seed=9)
    perm = np.random.default_rng(9).permutation(p.n_edges)
    gp, gq = _gpu_backward(p), _gpu_backward(q)
    # the per-edge output follows the caller's edge order
    assert rel_err(gq["grad_edge_vec"], gp["grad_edge_vec"][perm]) < 1e-5
    for k in ["grad_x", "grad_w", "grad_w_rad", "grad_b_rad"]:
        assert rel_err(gq[k], gp[k]) < 1e-5, k
    assert rel_err(_gpu_forward(q), _gpu_forward(p)) < 1e-5


def test_empty_graph_and_isolated_nodes():
    p = _small(L=2, M=1, C=16, n=20, nb=3, seed=10)
    e = dataclasses.replace(p, edge_index=np.zeros((2, 0), np.int64), edge_vec=np.zeros((0, 3)))
    assert float(_gpu_forward(e).abs().max()) == 0.0
    g = _gpu_backward(e)
    for k, t in g.items():
        assert float(t.abs().max()) == 0.0 if t.numel() else True, k
    keep = p.edge_index[1] != 0
    q = dataclasses.replace(p, edge_index=p.edge_index[:, keep], edge_vec=p.edge_vec[keep])
    out = _gpu_forward(q)
    assert float(out[0].abs().max()) == 0.0
    assert rel_err(out, oracle_forward(q)) < 1e-4


def test_device_reports_bad_index_and_zero_length_edge():
    p = _small(L=2, M=2, C=16, n=30, nb=4, seed=11)
    d = _dev(p)
    ei = d["edge_index"].clone()
    ei[1, 5] = p.n_nodes + 3
    B.forward(_desc(p), d["x"], ei, d["edge_vec"], d["w"], d["w_rad"], d["b_rad"])
    assert B.check(DEV) == 5
    ev = d["edge_vec"].clone()
    ev[7] = 0.0
    B.forward(_desc(p), d["x"], d["edge_index"], ev, d["w"], d["w_rad"], d["b_rad"])
    assert B.check(DEV) == 7
    B.forward(_desc(p), d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"], d["b_rad"])
    assert B.check(DEV) == 0


# ---------------------------------------------------------------------------
# double backward
# ---------------------------------------------------------------------------
DB_CASES = [
    ("tiny", lambda: synth.make_problem("tiny")),
    ("L3M2C32", lambda: _small(L=3, M=2, C=32, n=150, nb=20, seed=12)),
    ("L2M1C16_chunks", lambda: _small(L=2, M=1, C=16, n=600, nb=30, seed=13)),  # 18,000 edges
    ("L4M2C128_bf16", lambda: _small(L=4, M=2, C=128, n=60, nb=20, seed=14, bf16=True)),
]


def _gpu_double_backward(p, gg_x, gg_r):
    d = _dev(p)
    t = lambda a: None if a is None else torch.as_tensor(np.asarray(a)).float().to(DEV)  # noqa
    out = B.double_backward(_desc(p), d["x"], d["edge_index"], d["edge_vec"], d["w"],
                            d["w_rad"], d["b_rad"], d["grad_out"], gg_x=t(gg_x),
                            gg_edge_vec=t(gg_r))
    assert B.check(DEV) == 0
    return out


@pytest.mark.parametrize("which", ["r", "x", "rx"])
@pytest.mark.parametrize("name,make", DB_CASES, ids=[c[0] for c in DB_CASES])
def test_double_backward_parity(name, make, which):
    from helpers import oracle_double_backward
    p = make()
    rng = np.random.default_rng(21)
    gg_r = rng.standard_normal(p.edge_vec.shape) if "r" in which else None
    gg_x = rng.standard_normal(p.x.shape) if "x" in which else None
    got = _gpu_double_backward(p, gg_x, gg_r)
    ref = oracle_double_backward(p, gg_x=gg_x, gg_edge_vec=gg_r)
    for k in ["d_x", "d_w", "d_w_rad", "d_b_rad", "d_grad_out", "d_edge_vec"]:
        err = rel_err(got[k], ref[k])
        assert err < TOL[p.x_bf16], (name, which, k, err)


def test_force_training_step_parity():
    # energy = sum of l = 0 outputs; forces come from grad_edge_vec; a force
    # loss cotangent on grad_edge_vec is pulled back to the weights.
    p = synth.make_problem("force", seed=0, n_atoms=120, max_nb=20, lmax=3, mmax=2, c=32)
    g = _gpu_backward(p, need=["grad_edge_vec"])["grad_edge_vec"]
    ref = oracle_backward(p)["grad_edge_vec"]
    assert rel_err(g, ref) < 1e-4
    gg_r = np.random.default_rng(3).standard_normal(p.edge_vec.shape)
    got = _gpu_double_backward(p, None, gg_r)
    from helpers import oracle_double_backward
    want = oracle_double_backward(p, gg_edge_vec=gg_r)
    for k in ["d_w", "d_w_rad", "d_b_rad", "d_x", "d_edge_vec"]:
        assert rel_err(got[k], want[k]) < 1e-4, k


def test_chunk_size_does_not_change_results():
    # the same problem in one chunk and in 1,024-edge chunks
    p = _small(L=4, M=2, C=64, n=160, nb=24, seed=31)
    out1, g1 = _gpu_forward(p).cpu(), {k: v.cpu() for k, v in _gpu_backward(p).items()}
    try:
        assert B.set_max_chunk_edges(1000) == 1024
        out2, g2 = _gpu_forward(p).cpu(), {k: v.cpu() for k, v in _gpu_backward(p).items()}
    finally:
        B.set_max_chunk_edges(0)
    # only the summation order differs (reductions onto nodes, the K split of
    # the weight gradient); each order carries the split product's ~1e-5
    # relative error
    assert rel_err(out2, out1) < 5e-5
    for k in g1:
        assert rel_err(g2[k], g1[k]) < 5e-5, k


def test_preallocated_outputs():
    # results written into caller-given tensors equal freshly allocated ones
    p = _small(L=3, M=2, C=32, n=80, nb=12, seed=33)
    d = _dev(p)
    desc = _desc(p)
    ref = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                     d["b_rad"], d["grad_out"])
    given = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
    got = B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                     d["b_rad"], d["grad_out"], out=given)
    for k in ref:
        assert got[k].data_ptr() == given[k].data_ptr()
        assert rel_err(got[k], ref[k]) < 1e-6, k
    with pytest.raises(ValueError):
        B.backward(desc, d["x"], d["edge_index"], d["edge_vec"], d["w"], d["w_rad"],
                   d["b_rad"], d["grad_out"], out={"grad_x": torch.empty(3, device=DEV)})


def test_bounded_wait_reports_timeout_and_context_survives():
    # a wait that nothing completes gives up and reports SO2_ERR_TIMEOUT
    assert B.wait_selftest(DEV, limit_us=2000) == 6
    # the context is still usable: a small forward afterwards is correct
    p = synth.make_problem("tiny")
    assert rel_err(_gpu_forward(p), oracle_forward(p)) < 1e-4
