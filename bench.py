#!/usr/bin/env python
"""Throughput of the SO(2) edge convolution, forward + backward, on B200.

One step = so2conv_forward + so2conv_backward (all five gradients) over the
eSEN-like synthetic graph (2,000 atoms, periodic, 0.1 atoms/A^3, 30 nearest
neighbours within 6 A -> E = 60,000 edges; lmax 4, mmax 2, C 128, 16 RBFs,
f32).  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) the default (``--split dst``)
runs ONE graph of N times the workload's atoms (same density, so about N
times the edges) split over the ranks by destination node: each rank owns a
contiguous node range and the edges into it; node features are all-gathered
before the convolution, grad_x is reduce-scattered to its owners and the
weight gradients are all-reduced (NCCL).  Per-GPU work stays that of the
one-GPU workload ("weak" scaling).  ``--split replicas`` runs an independent
copy of the workload per rank instead (no collective on the data path).
The barrier and the max-over-ranks of the timed region bracket every step.
``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload on the host cores (rank 0 only).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from so_edge_convolution_b200 import synth  # noqa: E402

METRIC = "SO(2)-conv edges/sec (fwd+bwd, lmax=4, C=128) and % of roofline"
# name -> (synthetic problem, workload text, algorithmic products per step,
# products the kernels execute per step).  Algorithmic work counts one mixing
# product per forward, two per backward (the transposed product and the weight
# gradient) and three per double backward; the backward's recomputation of the
# forward product (it stores no per-edge tensor) is an implementation cost and
# is reported separately.
CONFIGS = {
    "esen": ("esen", "eSEN-like: N=2000 atoms periodic at 0.1/A^3, 30 nearest within 6 A "
             "(E=60000), lmax=4, mmax=2, C=128, 16 RBFs, f32 features and weights, "
             "forward+backward", 3, 4),
    "force": ("force", "force-training step on the eSEN-like graph: forward, backward to the "
              "edge vectors, force assembly and loss, double backward to the weights, f32", 5, 7),
    "md": ("force", "molecular-dynamics step on the eSEN-like graph: forward, backward to the "
           "edge vectors only and force assembly (no weight gradients), f32", 2, 3),
    "uma": ("uma", "UMA-like: N=5000 atoms, 30 nearest within 6 A (E=150000), lmax=6, mmax=2, "
            "C=128, bf16 features and weights, f32 accumulation, forward+backward", 3, 4),
    "large": ("large", "Large periodic: N=20000 atoms, 50 nearest within 6 A (E=1000000), "
              "lmax=4, mmax=2, C=128, bf16 features, f32 accumulation, forward+backward", 3, 4),
    "block": ("esen", "message block on the eSEN-like graph: two SO(2) convolutions with the "
              "edge-frame activation between them (E=60000, lmax=4, mmax=2, C=128, f32), "
              "forward+backward", 6, 8),
}
WORKLOAD = CONFIGS["esen"][1]
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


def mixing_flops_per_edge(L, M, ci, co):
    f = 2 * ((L + 1) * co) * ((L + 1) * ci)
    for m in range(1, M + 1):
        k = L + 1 - m
        f += 8 * (k * co) * (k * ci)
    return f


def kernel_sources_sha256():
    """Hash of the CUDA sources and the C header, to tell whether recorded
    counters still describe the kernels that are built now."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "so_edge_convolution_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for path in files + [os.path.join(ROOT, "include", "so2conv.h")]:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + b"\0" + f.read())
    return h.hexdigest()


def kernel_traffic(config):
    """The ncu record committed for this workload (DRAM bytes per launch of the
    mixing kernel, averaged over one step's launches); None when there is none
    or the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"gemm_tc_{config}_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("sources_sha256") != kernel_sources_sha256():
        return None
    return rec


def compulsory_bytes(config, p, n_nodes, n_edges):
    """Bytes of every input and output tensor of the step's library calls,
    each touched once per call (the HBM floor of the step), for calls over
    n_nodes node rows and n_edges edges."""
    S = (p.lmax + 1) ** 2
    xe = 2 if p.x_bf16 else 4
    we = 2 if p.w_bf16 else 4
    nw = sum(r * k for r, k in synth.weight_block_shapes(p.lmax, p.mmax, p.c_in, p.c_out))
    x = n_nodes * S * p.c_in * xe
    node_out = n_nodes * S * p.c_out * 4
    node_in = n_nodes * S * p.c_in * 4
    G = node_out
    ev = n_edges * 3 * 4
    rad = (p.n_rbf + 1) * p.c_out * 4
    shared = x + n_edges * 2 * 8 + ev + nw * we + rad
    fwd = shared + node_out
    if config == "md":
        return fwd + shared + G + ev
    if config == "block":  # a second weight set and gate, read and differentiated
        extra = nw * we + rad
        return fwd + extra + shared + extra + G + node_in + 2 * (nw * 4 + rad) + ev
    bwd = shared + G + node_in + nw * 4 + rad + ev
    if config == "force":
        bwd_r = shared + G + ev
        dbl = shared + G + ev + nw * 4 + rad
        return fwd + bwd_r + dbl
    return fwd + bwd


def step_traffic(config):
    """DRAM bytes (read + write) of every kernel of one step, from the ncu
    record committed for this workload; None when there is none or the
    kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"gemm_tc_{config}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("sources_sha256") != kernel_sources_sha256():
        return None
    return rec.get("dram_bytes_per_step_all_kernels")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.ident:
            cmd += ["-i", self.ident]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline object)
# ---------------------------------------------------------------------------
def oracle_sample_time(p, n_edges_sample, reps=1):
    import oracle as O
    torch.set_num_threads(os.cpu_count() or 1)
    sel = np.arange(min(n_edges_sample, p.n_edges))
    src = torch.from_numpy(p.edge_index[0, sel].copy())
    dst = torch.from_numpy(p.edge_index[1, sel].copy())
    vec = torch.from_numpy(p.edge_vec[sel].copy())
    desc = O.Desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff)
    args = (torch.from_numpy(p.x), src, dst, vec, torch.from_numpy(p.w),
            torch.from_numpy(p.w_rad), torch.from_numpy(p.b_rad), desc)
    G = torch.from_numpy(p.grad_out)
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        O.forward(*args)
        O.backward(*args, G)
        times.append(time.perf_counter() - t0)
    return len(sel), times, torch.get_num_threads()


def run_reference(args, world, rank):
    if rank != 0:
        return
    p = synth.make_problem("esen", seed=0)
    n = 512
    oracle_sample_time(p, n, reps=1)  # warm caches
    ts = []
    for _ in range(max(args.warmup, 0)):
        oracle_sample_time(p, n, reps=1)
    for _ in range(args.steps):
        _, t, cores = oracle_sample_time(p, n, reps=1)
        ts += t
    per_step = statistics.mean(ts)
    value = n / per_step
    sample = (f"first {n} edges (destination-major) of the eSEN-like graph per step, "
              "float64 oracle forward+backward on the host cores")
    line = {"metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample_edges_per_step": n},
            "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# One graph split by destination over the ranks
# ---------------------------------------------------------------------------
def dst_problem(prob, world, n_atoms=None, **overrides):
    """The job's graph: the workload's generator with world x its atoms (the
    periodic box grows with the atom count, so the density and the edges per
    atom stay those of the one-GPU workload).  n_atoms (per rank) and the
    other overrides shrink it for tests."""
    base = synth.CONFIGS[prob]["n_atoms"] if n_atoms is None else n_atoms
    return synth.make_problem(prob, seed=0, n_atoms=base * world, **overrides)


def dst_inputs(p, sg, xdt, wdt):
    """This rank's host inputs: its node rows of x and grad_out, its edges."""
    T = torch.from_numpy
    return {
        "x": sg.local_rows(T(p.x).to(xdt)),
        "edge_index": sg.edge_index.clone(),
        "edge_vec": sg.edge_vec.to(torch.float32).clone(),
        "w": T(p.w).to(wdt),
        "w_rad": T(p.w_rad.astype(np.float32)),
        "b_rad": T(p.b_rad.astype(np.float32)),
        "grad_out": sg.local_rows(T(p.grad_out.astype(np.float32))),
    }


def make_dst_step(sg, desc, op=None):
    """forward + backward of the rank's share (sharded.forward / backward)
    on the inputs in `t` (as dst_inputs lays them out)."""
    import copy
    from so_edge_convolution_b200 import sharded as S

    def step(t, o=None):
        v = copy.copy(sg)
        v.edge_index, v.edge_vec = t["edge_index"], t["edge_vec"]
        out = S.forward(v, desc, t["x"], t["w"], t["w_rad"], t["b_rad"], op=op)
        g = S.backward(v, desc, t["x"], t["w"], t["w_rad"], t["b_rad"], t["grad_out"], op=op)
        return out, g
    return step


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    from so_edge_convolution_b200 import binding as B
    from so_edge_convolution_b200 import build
    build.build()
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    B.set_max_chunk_edges(args.chunk_edges)
    prob, workload, n_products, n_executed = CONFIGS[args.config]
    split = args.split if args.split != "auto" else ("dst" if world > 1 else "replicas")
    if split == "dst" and world == 1:
        split = "replicas"  # one rank owns the whole graph
    if split == "dst" and args.config in ("force", "md", "block"):
        raise SystemExit("--split dst runs the forward + backward workloads")
    p = dst_problem(prob, world) if split == "dst" else synth.make_problem(prob, seed=rank)
    E = p.n_edges  # edges this rank's library calls process (set below for dst)
    bf16 = p.x_bf16
    xdt = torch.bfloat16 if bf16 else torch.float32
    wdt = torch.bfloat16 if bf16 else torch.float32
    desc = B.make_desc(p.lmax, p.mmax, p.c_in, p.c_out, p.n_rbf, p.rbf_cutoff,
                       B.SO2_BF16 if bf16 else B.SO2_F32)
    if args.config == "block":  # the second convolution's weights and gate
        rng2 = np.random.default_rng(1000 + rank)
        w2 = rng2.standard_normal(p.w.shape) * p.w.std()
        w_rad2 = rng2.standard_normal(p.w_rad.shape) / np.sqrt(p.n_rbf)
        b_rad2 = rng2.standard_normal(p.b_rad.shape) / np.sqrt(p.n_rbf)
    host = {
        "x": torch.from_numpy(p.x).to(xdt).pin_memory(),
        "edge_index": torch.from_numpy(p.edge_index).pin_memory(),
        "edge_vec": torch.from_numpy(p.edge_vec.astype(np.float32)).pin_memory(),
        "w": torch.from_numpy(p.w).to(wdt).pin_memory(),
        "w_rad": torch.from_numpy(p.w_rad.astype(np.float32)).pin_memory(),
        "b_rad": torch.from_numpy(p.b_rad.astype(np.float32)).pin_memory(),
        "grad_out": torch.from_numpy(p.grad_out.astype(np.float32)).pin_memory(),
        "f_ref": torch.from_numpy(p.f_ref.astype(np.float32)).pin_memory(),
    }
    if args.config == "block":
        host.update(w2=torch.from_numpy(w2).to(wdt).pin_memory(),
                    w_rad2=torch.from_numpy(w_rad2.astype(np.float32)).pin_memory(),
                    b_rad2=torch.from_numpy(b_rad2.astype(np.float32)).pin_memory())
    sg = None
    if split == "dst":
        from so_edge_convolution_b200 import sharded as S
        sg = S.ShardedGraph(torch.from_numpy(p.edge_index), torch.from_numpy(p.edge_vec),
                            p.n_nodes, rank, world)
        host = {k: v.pin_memory() for k, v in dst_inputs(p, sg, xdt, wdt).items()}
        E = int(sg.edge_ids.numel())
    E_job = p.n_edges if split == "dst" else world * E
    d = {k: v.to(dev) for k, v in host.items()}
    ws = B.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # o: optional preallocated results {"out": tensor, "g": {name: tensor}}
    def step_fwd_bwd(t, o=None):
        out = B.forward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                        t["b_rad"], ws=ws, out=o["out"] if o else None)
        g = B.backward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                       t["b_rad"], t["grad_out"], ws=ws, out=o["g"] if o else None)
        return out, g

    def step_force(t, o=None):
        # energy = sum of l = 0 outputs (its cotangent is grad_out), forces from
        # the edge-vector gradient, loss 1/2 |F - F_ref|^2 pulled back through
        # the double backward to the weights.
        out = B.forward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                        t["b_rad"], ws=ws, out=o["out"] if o else None)
        gr = B.backward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                        t["b_rad"], t["grad_out"], need=["grad_edge_vec"],
                        ws=ws)["grad_edge_vec"]
        src, dst = t["edge_index"][0], t["edge_index"][1]
        F = torch.zeros_like(t["f_ref"])
        F.index_add_(0, src, -gr).index_add_(0, dst, gr)
        dF = F - t["f_ref"]
        gg_r = dF[dst] - dF[src]
        g = B.double_backward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                              t["b_rad"], t["grad_out"], gg_edge_vec=gg_r,
                              need=["d_w", "d_w_rad", "d_b_rad"], ws=ws,
                              out=o["g"] if o else None)
        return out, g

    def step_md(t, o=None):
        # energy and forces: the forward, the edge-vector gradient of the
        # energy (cotangent grad_out) and F_i = sum of the edge gradients
        out = B.forward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                        t["b_rad"], ws=ws, out=o["out"] if o else None)
        g = B.backward(desc, t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"],
                       t["b_rad"], t["grad_out"], need=["grad_edge_vec"], ws=ws,
                       out=o["g"] if o else None)
        gr = g["grad_edge_vec"]
        src, dst = t["edge_index"][0], t["edge_index"][1]
        F = o["g"]["forces"].zero_() if o else torch.zeros_like(t["f_ref"])
        F.index_add_(0, src, -gr).index_add_(0, dst, gr)
        return out, {"grad_edge_vec": gr, "forces": F}

    def step_block(t, o=None):
        a = (t["x"], t["edge_index"], t["edge_vec"], t["w"], t["w_rad"], t["b_rad"], t["w2"],
             t["w_rad2"], t["b_rad2"])
        out = B.block_forward(desc, *a, ws=ws, out=o["out"] if o else None)
        g = B.block_backward(desc, *a, t["grad_out"], ws=ws, out=o["g"] if o else None)
        return out, g

    step = {"force": step_force, "md": step_md, "block": step_block}.get(args.config,
                                                                       step_fwd_bwd)
    if split == "dst":
        step = make_dst_step(sg, desc)
        ws = None  # the sharded calls use the binding's own per-device workspace

    torch.cuda.synchronize()
    resident = torch.cuda.memory_allocated(dev)  # inputs, flush buffer (before any step)
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(max(args.warmup, 3)):
        step(d)
    torch.cuda.synchronize()
    st = B.check(dev, ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    # device memory: the library's workspace per call (sized by the ABI) and the
    # peak torch allocation of a step above what was resident before it (the
    # workspace, the outputs and, for --split dst, the gathered node arrays)
    if args.config == "block":
        ws_sizes = {"block_forward": B.block_workspace_size(desc, int(d["x"].shape[0]), E, 0),
                    "block_backward": B.block_workspace_size(desc, int(d["x"].shape[0]), E, 1)}
    else:
        n_call = sg.n_pad if sg is not None else p.n_nodes
        ws_sizes = {k: B.workspace_size(desc, n_call, E, w) for k, w in
                    (("forward", B.WS_FORWARD), ("backward", B.WS_BACKWARD),
                     ("double_backward", B.WS_DOUBLE_BACKWARD))}
    memory = {"workspace_bytes": ws_sizes,
              "peak_step_bytes_above_inputs": int(torch.cuda.max_memory_allocated(dev) - resident),
              "chunk_edges": int(B.load().so2conv_max_chunk_edges()),
              "note": "no tensor of E x (lmax+1)^2 x C is allocated; per-edge intermediates "
                      "live in the workspace for one chunk of edges at a time"}

    # ---- device-resident timed region ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    B.profile_enable(True)
    launches0 = B.launch_count()
    for k in range(args.steps):
        flush.zero_()  # evict L2 between steps (outside the timed events)
        starts[k].record()
        step(d)
        ends[k].record()
    torch.cuda.synchronize()
    launches = B.launch_count() - launches0  # this library's kernels, all timed steps
    B.profile_enable(False)
    prof = B.profile_read()
    clk = clocks.stop() if clocks else None
    barrier(world)
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = E_job * args.steps / (total_ms * 1e-3)

    # ---- roofline (algorithmic mixing FLOPs only: the recomputed product is not counted) ----
    # The bound is the tensor-core one (compulsory bytes are ~30x below it).
    # Peaks: the burst bf16 figure applies (the timed region is ~0.1 s, not a
    # seconds-long loop); the f32 path is held against the TF32-equivalent
    # peak (nominal dense TF32 / BF16 = 1.1 / 2.25), the bf16 path against
    # bf16.  The sustained figures are printed beside them.
    pk, src = peaks()
    fpe = mixing_flops_per_edge(p.lmax, p.mmax, p.c_in, p.c_out)
    n_gemm = sum(prof[k][0] for k in B.TENSOR_KINDS)
    gemm_ms = sum(prof[k][1] for k in B.TENSOR_KINDS)
    alg_flops = float(n_products) * fpe * E * args.steps
    achieved = alg_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    tf32_ratio = 1.0 if bf16 else 1.1 / 2.25
    peak_tf = pk["bf16_tflops"] * tf32_ratio
    peak_tf_sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * tf32_ratio
    step_tflops = alg_flops / (total_ms * 1e-3) / 1e12
    cbytes = compulsory_bytes(args.config, p, sg.n_pad if sg is not None else p.n_nodes, E)
    t_roof_ms = max(n_products * fpe * E / (peak_tf * 1e12),
                    cbytes / (pk["hbm_gbs"] * 1e9)) * 1e3
    # the committed DRAM record was taken with the library's default chunk
    traffic = kernel_traffic(args.config) if args.chunk_edges == 0 else None
    step_dram = step_traffic(args.config) if args.chunk_edges == 0 else None
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": (achieved / peak_tf) if achieved else None,
                "traffic": traffic.get("dram_bytes_per_launch") if traffic else None,
                "kernel": ("k_gemm_tc (bf16, f32 accumulate)" if bf16 else
                           "k_gemm_tc (split-bf16 x3, f32 accumulate)"),
                "peak_basis": (f"{src} bf16 burst" if bf16 else
                               f"{src} bf16 burst x nominal TF32/BF16 ratio 1.1/2.25"),
                "frac_vs_sustained": (achieved / peak_tf_sus) if achieved else None,
                "products_per_step": n_products,
                "executed_products_per_step": n_executed,
                "algorithmic_gflop_per_step": n_products * fpe * E / 1e9,
                "gemm_launches_per_step": n_gemm / args.steps,
                "gemm_ms_per_step": gemm_ms / args.steps,
                "step_roofline_frac": step_tflops / peak_tf,
                "step_roofline_frac_vs_sustained": step_tflops / peak_tf_sus,
                "roofline_ms_per_step": t_roof_ms,
                "compulsory_bytes_per_step": cbytes,
                "dram_bytes_per_step": step_dram,
                "traffic_over_compulsory": (step_dram / cbytes) if step_dram else None}
    # where the step's time goes: CUDA events around every launch group, in a
    # few extra steps after the timed ones (so they add nothing to its time)
    n_bd = 3
    torch.cuda.synchronize()
    B.profile_enable(True, all_kinds=True)
    for _ in range(n_bd):
        flush.zero_()
        step(d)
    torch.cuda.synchronize()
    B.profile_enable(False)
    breakdown = {B.PROFILE_KINDS[k]: round(v[1] / n_bd, 4) for k, v in B.profile_read().items()}

    # ---- end to end through the C ABI from pinned host buffers ----
    # Every step copies its inputs from pinned host memory and its results back
    # to pinned host memory inside the timed region.  The copies run on their
    # own streams into double-buffered device inputs, so step k+1's upload and
    # step k-1's download overlap step k's kernels (as a prefetching loader
    # would); events order each buffer's reuse.
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dbufs = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in host.items()}
             for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    # untimed: one step per slot on filled inputs, whose results become the
    # slot's preallocated device results; pinned host buffers for them
    outs_dev, outs_host = [None, None], [None, None]
    for sl in range(2):
        for name, v in host.items():
            dbufs[sl][name].copy_(v)
        out0, g0 = step(dbufs[sl])
        outs_dev[sl] = {"out": out0, "g": g0}
        res = [out0] + [g0[kk] for kk in sorted(g0)]
        outs_host[sl] = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in res]
    e2e_s = torch.cuda.Event(enable_timing=True)
    e2e_e = torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    barrier(world)
    torch.cuda.synchronize()
    e2e_s.record(comp)
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    d2h = 0
    for k in range(n_e2e):
        sl = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_done[sl])  # step k-2 no longer reads these inputs
            for name, v in host.items():
                dbufs[sl][name].copy_(v, non_blocking=True)
            ev_in[sl].record(s_in)
        comp.wait_event(ev_in[sl])
        if k >= 2:
            comp.wait_event(ev_out[sl])  # step k-2's results are downloaded
        out, g = step(dbufs[sl], outs_dev[sl])
        ev_done[sl].record(comp)
        res = [out] + [g[kk] for kk in sorted(g)]
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[sl])
            for hbuf, r in zip(outs_host[sl], res):
                hbuf.copy_(r, non_blocking=True)
            ev_out[sl].record(s_out)
        d2h = sum(r.numel() * r.element_size() for r in res)
    comp.wait_stream(s_out)
    e2e_e.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e2e_s.elapsed_time(e2e_e), world, dev) / n_e2e
    e2e = {"value": E_job / (e2e_ms * 1e-3), "unit": "edges/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "copies": "pinned host buffers, every step, on copy streams overlapping the "
                     "neighbouring steps' kernels"}

    # ---- CPU oracle on a bounded sample (rank 0, one GPU only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "esen":
        n, ts, cores = oracle_sample_time(p, 2048, reps=3)
        cpu = {"value": n / statistics.median(ts), "unit": "edges/s", "cores": cores,
               "kind": "oracle",
               "sample": f"first {n} edges (destination-major) of the same graph, float64 "
                         "oracle forward+backward, median of 3 timed runs"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "edges/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if bf16 else "f32", "data": "synthetic",
                "config": {"workload": workload if split != "dst" else
                           workload + f"; one graph of {world} x the atoms split by destination",
                           "edges": E_job, "edges_per_rank": E, "nodes": p.n_nodes,
                           "l2": "flushed between timed steps (256 MB write)",
                           "chunk_edges": int(B.load().so2conv_max_chunk_edges()),
                           "parallelism": (f"dst-split x{world} (all-gather x, reduce-scatter "
                                           "grad_x, all-reduce grad_W; NCCL)" if split == "dst"
                                           else f"replicas x{world}" if world > 1 else "single")},
                "step_roofline_frac": roofline["step_roofline_frac"],
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "gpu_launches_per_step": launches // max(args.steps, 1),
                "clocks": clk, "breakdown_ms_per_step": breakdown, "memory": memory}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="esen",
                    help="workload (the headline line is esen; the others are for study)")
    ap.add_argument("--split", choices=["auto", "dst", "replicas"], default="auto",
                    help="N > 1: one graph split by destination (dst, the default) or "
                         "independent replicas")
    ap.add_argument("--chunk-edges", type=int, default=0,
                    help="edges per chunk of per-edge intermediates (0: the library's "
                         "default, 65,536)")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
