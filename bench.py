#!/usr/bin/env python3
"""Benchmark of the streaming CG tensor-product convolution on B200.

One step = one pass of the whole hot path over one synthetic batch of the
mace-like layer (4096 atoms in a periodic box at 0.1 atoms/A^3, all pairs within
5 A, 64x0e+64x1o+64x2e -> same, SH l<=3, R=8 Bessel radial basis): sender-sorted
graph view, forward, backward (dx, dTheta, dvec) and double backward in the
force-training shape (gg_x, gg_vec given, gg_Theta = 0) -> d_g, d_x, d_vec,
d_Theta.  The headline value is edges per second of that step; the same line
carries edges/s of the forward alone, of forward + backward and of the double
backward alone.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --suite [--steps K]    # one line per workload of the metric

N > 1 runs under torch.distributed.run: every rank processes its own graph
(seed = rank) with no collective on the data path (weak scaling); the step time
is the max over ranks.  --impl reference times the CPU oracle (the
conventional schedule) on bounded samples of the same workload, one process
per host core (the pages ship no runnable reference).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

WORKLOADS = {
    "mace": ("mace-like layer: 4096 atoms, periodic cube at 0.1 atoms/A^3, 5 A radius graph, "
             "64x0e+64x1o+64x2e -> 64x0e+64x1o+64x2e, SH l<=3, R=8 Bessel"),
    "capacity": ("capacity run of the mace-like layer: 1222309 atoms, periodic cube at 0.1 atoms/A^3 "
                 "(side 230.35 A), 5 A radius graph (~64 M edges), 64x0e+64x1o+64x2e, SH l<=3, R=8 Bessel; "
                 "receiver chunks of the workspace cap"),
    "sweep": ("edge-scaling sweep: 20000 nodes, periodic cube sized for mean degree {d:g}, 5 A radius graph, "
              "32x0e+32x1o+32x2e, SH l<=2, R=8 Bessel"),
    "wide": ("wide operator: 8192 nodes, mean degree 32, 5 A radius graph, 128x0e+128x1o+128x2e+128x3o, "
             "SH l<=3, R=8 Bessel"),
    "tiny": "tiny: 64 nodes, 512 random edges, 8x0e+8x1o, SH l<=2, R=4 Gaussian",
}


def workload(args):
    w = WORKLOADS[args.config].format(d=args.degree or 25)
    return w + ", channel-wise weights" if args.family == "channelwise" else w
METRIC = "edges/s (fwd + bwd + double bwd step)"
L2_BYTES = 126 * 1024 * 1024
FP32_LANES_PER_SM = 128
N_SM = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="mace")
    ap.add_argument("--gemm", default="fp32", choices=["fp32", "tf32", "simt"])
    ap.add_argument("--family", default="full", choices=["full", "channelwise"],
                    help="operator family: fully connected or channel-wise per-path weights")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--suite", action="store_true",
                    help="one JSON line per workload (tiny, mace, sweep d=25/100/400, wide fp32/tf32): "
                         "fwd, fwd+bwd and double-bwd edges/s, peak memory, roofline of the dominant kernel")
    ap.add_argument("--suite-configs", default="tiny,mace,sweep25,sweep100,sweep400,wide_fp32,wide_tf32",
                    help="comma-separated suite entries (also: capacity)")
    ap.add_argument("--shard", action="store_true",
                    help="with N > 1: one graph sharded over the ranks by receiver ranges (all-gather of x, "
                         "reduce-scatter of dx / d_x, all-reduce of the Theta gradients over NCCL; strong "
                         "scaling) instead of one independent graph per rank")
    ap.add_argument("--parity-sample", type=int, default=0,
                    help="after the timed steps, check the step's outputs against the oracle on this many sampled "
                         "receivers (out, d_g), senders (dx, d_x) and edges (dvec, d_vec), and dTheta / d_Theta "
                         "by additivity over two receiver halves of the graph; prints a second JSON line")
    ap.add_argument("--oracle-procs", type=int, default=0,
                    help="processes of the CPU oracle baseline (default: the host cores, at most 32)")
    ap.add_argument("--degree", type=float, default=None, help="mean degree of the sweep workload")
    ap.add_argument("--clock-log", default=None,
                    help="file for the nvidia-smi clock samples of the timed region ({rank} is replaced); "
                         "default: a temporary file")
    ap.add_argument("--workspace-cap", type=int, default=None,
                    help="bytes of node-side state per receiver chunk (default: none; 8 GiB for capacity)")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work model (per edge), from the plan's path table and CG pattern
# ---------------------------------------------------------------------------
def sources_digest(files):
    """Digest of the named CUDA/C++ sources of a kernel: counters taken on other sources do not apply."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "equivariant_gnn_tensor_receiver_b200", "csrc")
    for f in sorted(files):
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def work_model(T, plan):
    R = plan.R
    nnz_cache = {}
    fw = bw_r = bw_s = db_a = db_r = db_s = 0
    for p in plan.paths:
        key = (p["l1"], p["l2"], p["l3"])
        if key not in nnz_cache:
            C = T.tpconv_cg_coefficients(*key)
            nz = np.abs(C) > 0
            nnz_cache[key] = (int(nz.sum()), int(nz.any(axis=1).sum()))
        nnz, mnz = nnz_cache[key]
        n1, n3 = 2 * p["l1"] + 1, 2 * p["l3"] + 1
        ci, co = p["c_in"], p["c_out"]
        fw += nnz + ci * (mnz + R * n3)                           # M_e, M x, b (x) T
        bw_r += 2 * nnz + ci * (2 * mnz + 2 * R * n3)             # M_e; M x, dT, db, Q += x (x) dT; C : Q
        bw_s += nnz + co * (mnz + R * n1)                         # M_e, M^T g, b (x) U
        db_a += 2 * nnz + ci * (3 * mnz + 2 * R * n3)             # A1 only: A0 serves gg_Theta, absent here
        # M, Md; 3 M-products, 3 Q updates; C : Qw, Qh.  The step has no gg_Theta, so the
        # G~ terms (b G~ into dX, G~ . T0 into wb; 2 R n3 per channel) are not part of it.
        db_r += 4 * nnz + ci * (6 * mnz + 4 * R * n3)
        db_s += 2 * nnz + co * (2 * mnz + 3 * R * n1)
    return {"fwd_edge": fw, "bwd_edge_r": bw_r, "bwd_edge_s": bw_s, "dbl_edge_a": db_a, "dbl_edge_r": db_r,
            "dbl_edge_s": db_s}


def gemm_flops(plan_info, N):
    """Node-level Theta contractions per step (FMAs): out, G, dx, dTheta, d_g, d_x, d_Theta."""
    per = plan_info["mix_fma_per_node"]
    return {"fwd_node": per * N, "bwd_node_g": per * N, "bwd_node_x": 2 * per * N, "dbl_node_a": per * N,
            "dbl_node_x": 2 * per * N}


class ClockSampler:
    def __init__(self, index, path):
        self.path = path
        self.proc = None
        self.index = index

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        try:
            rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        except OSError:
            rows = []
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        mx = [float(r[2]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": reasons, "samples": len(rows)}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def theta_segments(paths, R, family):
    """Normal Theta blocks per path: R x C_in x C_out (std 1/sqrt(R C_in)) or R x C (std 1/sqrt(R))."""
    get = (lambda p, k: p[k]) if isinstance(paths[0], dict) else (lambda p, k: getattr(p, k))
    if family == "channelwise":
        return [(R * get(p, "c_in"), 1 / np.sqrt(R)) for p in paths]
    return [(R * get(p, "c_in") * get(p, "c_out"), 1 / np.sqrt(R * get(p, "c_in"))) for p in paths]


def oracle_sample(cfg, graph, n_recv, seed=100, family="full"):
    """Oracle step (fwd + bwd + double bwd) on the edges of the first n_recv receivers."""
    from oracle import conv
    c = W.CONFIGS[cfg]
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                        tuple(c["radial_params"]), family=family)
    rowptr, col, vec = graph
    e1 = int(rowptr[n_recv])
    rp = np.asarray(rowptr[:n_recv + 1], dtype=np.int64)
    # only the sample's receivers (first, keeping their numbers) and senders hold features
    nodes = np.unique(np.concatenate([np.arange(n_recv), np.asarray(col[:e1], dtype=np.int64)]))
    col = np.searchsorted(nodes, np.asarray(col[:e1], dtype=np.int64)).astype(np.int32)
    vec = vec[:e1]
    N = len(nodes)
    x = W.normal((N, prob.dim_in), seed)
    th = W.theta(theta_segments(prob.paths, prob.R, family), seed + 1)
    g = np.zeros((n_recv, prob.dim_out))
    g[:] = W.normal((n_recv, prob.dim_out), seed + 2)
    ggx = W.normal((N, prob.dim_in), seed + 3)
    ggv = W.normal((e1, 3), seed + 4)

    def step():
        send = np.asarray(col[:e1], dtype=np.int64)
        recv = conv.receivers_of(rp)
        Y, b = conv.geometry(prob, vec[:e1])
        conv.forward_core(prob, n_recv, send, recv, x, Y, b, th)
        conv.backward(prob, rp, col[:e1], vec[:e1], x, th, g)
        conv.double_backward(prob, rp, col[:e1], vec[:e1], x, th, g, ggx, ggv, None)

    return step, e1


def _oracle_proc(cfg, family, r0, n_recv, warmup, steps, ready, start, out):
    """One process of the parallel oracle baseline: the oracle step on the
    edges of receivers r0 .. r0+n_recv-1 (single-threaded BLAS), `warmup`
    untimed steps, then `steps` timed ones once every process is ready."""
    graph = W.graph_for(cfg, 0)
    rowptr, col, vec = graph
    # the sample: receivers r0.. renumbered to 0.. (their senders keep their own rows)
    e0, e1 = int(rowptr[r0]), int(rowptr[r0 + n_recv])
    rp = np.asarray(rowptr[r0:r0 + n_recv + 1], dtype=np.int64) - e0
    sub = (rp, np.asarray(col[e0:e1]), vec[e0:e1])
    step, e = oracle_sample(cfg, sub, n_recv, seed=100 + r0, family=family)
    for _ in range(warmup):
        step()
    ready.put(os.getpid())
    start.wait()
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    out.put((e, times))


def parallel_oracle(cfg, family, procs, n_recv, warmup, steps):
    """The CPU oracle (fp64 numpy, conventional schedule) timed on `procs`
    processes at once, each on its own block of n_recv receivers of the
    workload's graph.  Processes start with 'spawn' (never forked from a
    process that has used the GPU) and run with one BLAS thread each, so
    `procs` is the number of host cores busy.  Returns edges/s of all processes
    together over the slowest process's time, per step."""
    import multiprocessing as mp
    env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in env:
        os.environ[k] = "1"
    try:
        ctx = mp.get_context("spawn")
        ready, out, start = ctx.Queue(), ctx.Queue(), ctx.Event()
        ps = [ctx.Process(target=_oracle_proc, args=(cfg, family, i * n_recv, n_recv, warmup, steps, ready, start, out))
              for i in range(procs)]
        for p in ps:
            p.start()
        for _ in ps:
            ready.get(timeout=900)
        start.set()
        res = [out.get(timeout=3600) for _ in ps]
        for p in ps:
            p.join()
    finally:
        for k, v in env.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    edges = sum(e for e, _ in res)
    per_step = [max(t[i] for _, t in res) for i in range(steps)]
    dt = sum(per_step) / steps
    return {"value": edges / dt, "unit": "edges/s", "cores": procs, "kind": "oracle", "ms_per_step": dt * 1e3,
            "edges_per_step": edges,
            "sample": f"fp64 numpy oracle step (fwd + bwd + double bwd, conventional schedule) on {procs} "
                      f"processes x {n_recv} receivers ({edges} edges per step, one BLAS thread each), "
                      f"{steps} timed steps"}


def _sub_problem(rowptr, col, edges, include=()):
    """The listed edges (CSR positions) as a graph of their own: local receivers
    (sorted) first, then senders that are not receivers and the `include`d
    nodes that neither (isolated ones keep empty segments); returns
    (rowptr, col, edge ids in local CSR order, receivers' global ids, all local
    nodes' global ids)."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    recv_all = np.repeat(np.arange(len(rowptr) - 1), np.diff(rowptr))
    edges = np.sort(np.asarray(edges, dtype=np.int64))
    r = recv_all[edges]
    s = np.asarray(col, dtype=np.int64)[edges]
    recvs = np.unique(r)
    extra = np.setdiff1d(np.union1d(np.unique(s), np.asarray(include, dtype=np.int64)), recvs)
    nodes = np.concatenate([recvs, extra])
    pos = {int(g): i for i, g in enumerate(nodes)}
    lr = np.fromiter((pos[int(v)] for v in r), dtype=np.int64, count=len(r))
    lc = np.fromiter((pos[int(v)] for v in s), dtype=np.int64, count=len(s))
    order = np.argsort(lr, kind="stable")
    lrp = np.concatenate([[0], np.cumsum(np.bincount(lr, minlength=len(nodes)))])
    return lrp, lc[order], edges[order], recvs, nodes


def _parity_worker(job):
    """One oracle job of the parity check: (kind, config, family, arrays) -> arrays."""
    kind, cfg, family, a = job
    from oracle import conv
    c = W.CONFIGS[cfg]
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                        tuple(c["radial_params"]), family=family)
    rp, col, vec, x, th, g = a["rowptr"], a["col"], a["vec"], a["x"], a["theta"], a["g"]
    if kind == "recv":
        out = conv.forward(prob, rp, col, vec, x, th)
        return {"out": out}
    if kind == "recv_dbl":
        r = conv.double_backward(prob, rp, col, vec, x, th, g, a["gg_x"], a["gg_vec"], None)
        return {"d_g": r["d_g"]}
    if kind == "send":
        return {"dx": conv.backward(prob, rp, col, vec, x, th, g)["dx"]}
    if kind == "send_dbl":
        r = conv.double_backward(prob, rp, col, vec, x, th, g, a["gg_x"], a["gg_vec"], None)
        return {"d_x": r["d_x"]}
    if kind == "edge":
        rb = conv.backward(prob, rp, col, vec, x, th, g)
        r = conv.double_backward(prob, rp, col, vec, x, th, g, a["gg_x"], a["gg_vec"], None)
        return {"dvec": rb["dvec"], "d_vec": r["d_vec"]}
    raise ValueError(kind)


def sampled_parity(cfg, family, graph, inputs, out_rows, procs, k, seed=12345):
    """Element-wise parity of sampled rows against the oracle, on sub-graphs
    the oracle computes exactly: out and d_g of k (k/4) sampled receivers from
    their in-edges, dx and d_x of sampled senders from their out-edges, dvec
    and d_vec of sampled edges from the edge alone (with its receiver).
    inputs: host arrays x, theta, g, gg_x, gg_vec, vec (fp32 as the device
    holds them); out_rows(key, idx) -> the device result's rows idx (fp64).
    Returns the max-norm relative error per output."""
    import multiprocessing as mp
    rowptr, col, _ = graph
    rp64 = np.asarray(rowptr, dtype=np.int64)
    col64 = np.asarray(col, dtype=np.int64)
    N, E = len(rp64) - 1, len(col64)
    x, g, ggx, ggv, v32 = (inputs[key] for key in ("x", "g", "gg_x", "gg_vec", "vec"))
    th = np.asarray(inputs["theta"], dtype=np.float64)
    f64 = lambda a: np.asarray(a, dtype=np.float64)
    rng = np.random.default_rng(seed)
    k = min(k, N, E)
    k_dbl = max(1, k // 4)
    rs = np.sort(rng.choice(N, k, replace=False))
    ss = np.sort(rng.choice(N, k, replace=False))
    es = np.sort(rng.choice(E, k, replace=False))

    def job(kind, edges, include=()):
        lrp, lc, eids, recvs, nodes = _sub_problem(rowptr, col, edges, include)
        a = {"rowptr": lrp, "col": lc, "vec": f64(v32[eids]), "x": f64(x[nodes]), "theta": th,
             "g": f64(g[nodes]), "gg_x": f64(ggx[nodes]), "gg_vec": f64(ggv[eids])}
        return (kind, cfg, family, a), (recvs, nodes, eids)

    def edges_of_recv(r):
        return np.concatenate([np.arange(rp64[i], rp64[i + 1]) for i in r]) if len(r) else np.zeros(0, np.int64)

    def edges_of_send(sn):
        return np.nonzero(np.isin(col64, sn))[0]

    split = lambda arr, n: [a for a in np.array_split(arr, n) if len(a)]
    jobs, meta = [], []
    for kind, nodes_k, edges_of in (("recv", rs, edges_of_recv), ("recv_dbl", rs[:k_dbl], edges_of_recv),
                                    ("send", ss, edges_of_send), ("send_dbl", ss[:k_dbl], edges_of_send)):
        for part in split(nodes_k, procs):
            j, m = job(kind, edges_of(part), part)
            jobs.append(j)
            meta.append((kind, part, m))
    for part in split(es, procs):
        j, m = job("edge", part)
        jobs.append(j)
        meta.append(("edge", part, m))
    env = {key: os.environ.get(key) for key in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for key in env:
        os.environ[key] = "1"
    try:
        with mp.get_context("spawn").Pool(procs) as pool:
            results = pool.map(_parity_worker, jobs, chunksize=1)
    finally:
        for key, v in env.items():
            if v is None:
                os.environ.pop(key, None)
            else:
                os.environ[key] = v
    ref = {key: [] for key in ("out", "d_g", "dx", "d_x", "dvec", "d_vec")}
    got = {key: [] for key in ref}
    for (kind, part, (recvs, nodes, eids)), res in zip(meta, results):
        if kind in ("recv", "recv_dbl", "send", "send_dbl"):
            pos = {int(v): i for i, v in enumerate(nodes)}
            rows = np.array([pos[int(v)] for v in part])
            key = {"recv": "out", "recv_dbl": "d_g", "send": "dx", "send_dbl": "d_x"}[kind]
            ref[key].append(res[key][rows])
            got[key].append(out_rows(key, part))
        else:
            order = np.argsort(eids)  # back to the sampled (sorted) edge order
            for key in ("dvec", "d_vec"):
                ref[key].append(res[key][order])
                got[key].append(out_rows(key, np.sort(eids)))
    errs = {}
    for key in ref:
        rr, gg = np.concatenate(ref[key]), np.concatenate(got[key])
        errs[key] = float(np.abs(gg - rr).max() / max(np.abs(rr).max(), 1e-30))
    return errs, dict(receivers=k, senders=k, edges=k, dbl_nodes=k_dbl)


def parity_check(args, work, graph, procs, k):
    """Sampled parity of one full step of the workload against the oracle (see
    --parity-sample), plus dTheta / d_Theta by additivity over receiver halves."""
    import torch
    N = work.N
    rp64 = np.asarray(graph[0], dtype=np.int64)
    # host inputs stay fp32 views of the pinned buffers; only sampled rows of
    # the outputs come back from the device (the capacity workload's full
    # arrays are tens of GB)
    h = {key: v.numpy() for key, v in work.host.items()}

    def gpu_rows(key, idx):
        t = work.outs[key]
        return t.index_select(0, torch.as_tensor(idx, dtype=torch.int64, device=t.device)).double().cpu().numpy()

    t0 = time.perf_counter()
    errs, sampled = sampled_parity(args.config, args.family, graph, h, gpu_rows, procs, k)
    gpu = {key: work.outs[key].double().cpu().numpy() for key in ("dtheta", "d_theta")}
    # dTheta and d_Theta: the full graph against the sum over its two receiver
    # halves (the library on both sides; additivity holds at any size)
    T = work.T
    half = N // 2
    sums = {}
    d = work.d
    for lo, hi in ((0, half), (half, N)):
        sub_rp = np.concatenate([np.zeros(lo, np.int64), rp64[lo:hi + 1] - rp64[lo],
                                 np.full(N - hi, rp64[hi] - rp64[lo], np.int64)])
        e0, e1 = int(rp64[lo]), int(rp64[hi])
        Gs = T.Graph(torch.as_tensor(sub_rp, dtype=torch.int32, device=work.dev), d["col"][e0:e1],
                     d["vec"][e0:e1])
        a = T.backward(work.plan, Gs, d["x"], d["theta"], d["g"], want=("dtheta",))["dtheta"]
        b = T.double_backward(work.plan, Gs, d["x"], d["theta"], d["g"], d["gg_x"], d["gg_vec"][e0:e1], None,
                              want=("d_theta",))["d_theta"]
        torch.cuda.synchronize()
        sums["dtheta"] = sums.get("dtheta", 0.0) + a.double().cpu().numpy()
        sums["d_theta"] = sums.get("d_theta", 0.0) + b.double().cpu().numpy()
        del Gs, a, b
        torch.cuda.empty_cache()
    for key in ("dtheta", "d_theta"):
        errs[key + "_additivity"] = float(np.abs(sums[key] - gpu[key]).max() / max(np.abs(gpu[key]).max(), 1e-30))
    tol = 1e-5 if args.gemm in ("fp32", "simt") else 5e-3
    return {"parity": args.config, "gemm": args.gemm, "family": args.family, "nodes": N, "edges": work.E,
            "sampled_receivers": sampled["receivers"], "sampled_senders": sampled["senders"],
            "sampled_edges": sampled["edges"], "sampled_dbl_nodes": sampled["dbl_nodes"],
            "max_norm_rel_err": errs, "tolerance": tol, "pass": all(v < tol for v in errs.values()),
            "oracle_s": round(time.perf_counter() - t0, 1), "oracle_procs": procs}


def reduce_over_ranks(v, op, world, device):
    """Max or sum of a per-rank scalar over the default process group (any
    backend: nccl with a CUDA device, gloo with the CPU); identity at world 1."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(edges_local, step_ms_local, world, device):
    """Whole-job edges/s of independent per-rank graphs: the edges of all ranks
    over the slowest rank's step time (device time, max over ranks)."""
    step_ms = reduce_over_ranks(step_ms_local, "max", world, device)
    edges = reduce_over_ranks(float(edges_local), "sum", world, device)
    return edges / (step_ms * 1e-3), step_ms, edges


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    procs = args.oracle_procs or min(32, host_cores())
    r = parallel_oracle(args.config, args.family, procs, 4, max(1, min(args.warmup, 1)), args.steps)
    v = r["value"]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload(args), "sample": r["sample"]},
            "cpu_baseline": {k: r[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": v, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class Work:
    """One workload resident on the device: plan, inputs, outputs, workspaces
    and the library calls of one step (all arithmetic in the CUDA library)."""

    def __init__(self, T, L, config, graph, gemm, family, cap, dev, seed=0):
        import torch
        c = W.CONFIGS[config]
        self.T, self.L, self.dev, self.cap = T, L, dev, cap
        rowptr, col, vec = graph
        self.N, self.E = N, E = len(rowptr) - 1, len(col)
        self.plan = plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                                  radial_params=c["radial_params"], gemm=gemm, workspace_cap=cap, family=family)
        f32 = torch.float32
        pin = lambda a, dt=f32: torch.as_tensor(np.ascontiguousarray(a), dtype=dt).pin_memory()
        self.host = {
            "rowptr": pin(rowptr, torch.int32), "col": pin(col, torch.int32), "vec": pin(vec),
            "x": pin(W.normal((N, plan.dim_in), 10 + seed)),
            "theta": pin(W.theta(theta_segments(plan.paths, plan.R, family), 11 + seed)),
            "g": pin(W.normal((N, plan.dim_out), 12 + seed)),
            "gg_x": pin(W.normal((N, plan.dim_in), 13 + seed)),
            "gg_vec": pin(W.normal((E, 3), 14 + seed)),
        }
        self.d = {k: v.to(dev) for k, v in self.host.items()}
        self.outs = {
            "out": torch.empty(N, plan.dim_out, device=dev), "dx": torch.empty(N, plan.dim_in, device=dev),
            "dtheta": torch.empty(plan.theta_numel, device=dev), "dvec": torch.empty(E, 3, device=dev),
            "d_g": torch.empty(N, plan.dim_out, device=dev), "d_x": torch.empty(N, plan.dim_in, device=dev),
            "d_vec": torch.empty(E, 3, device=dev), "d_theta": torch.empty(plan.theta_numel, device=dev),
        }
        self.perm = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
        self.s_rowptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
        self.s_recv = torch.empty(max(E, 1), dtype=torch.int32, device=dev)
        self.ws = {op: T.workspace(plan, op, N, E, dev) for op in (L.OP_FORWARD, L.OP_BACKWARD,
                                                                   L.OP_DOUBLE_BACKWARD, L.OP_TRANSPOSE)}
        self.ws_bytes = sum(w.numel() for w in self.ws.values())

    def transpose(self, src=None):
        src, L = src or self.d, self.L
        L.tpconv_graph_transpose(self.plan, self.N, self.E, src["rowptr"], src["col"], self.perm, self.s_rowptr,
                                 self.s_recv, self.ws[L.OP_TRANSPOSE])

    def fwd(self, src=None, outs=None):
        src, L, o = src or self.d, self.L, outs or self.outs
        L.tpconv_forward(self.plan, self.N, self.E, src["rowptr"], src["col"], src["vec"], src["x"], src["theta"],
                         o["out"], self.ws[L.OP_FORWARD])

    def bwd(self, src=None, outs=None):
        src, L, o = src or self.d, self.L, outs or self.outs
        L.tpconv_backward(self.plan, self.N, self.E, src["rowptr"], src["col"], self.perm, self.s_rowptr,
                          self.s_recv, src["vec"], src["x"], src["theta"], src["g"], o["dx"], o["dtheta"], o["dvec"],
                          None, None, self.ws[L.OP_BACKWARD])

    def dbl(self, src=None, outs=None):
        src, L, o = src or self.d, self.L, outs or self.outs
        L.tpconv_double_backward(self.plan, self.N, self.E, src["rowptr"], src["col"], self.perm, self.s_rowptr,
                                 self.s_recv, src["vec"], src["x"], src["theta"], src["g"], src["gg_x"],
                                 src["gg_vec"], None, o["d_g"], o["d_x"], o["d_vec"], o["d_theta"],
                                 self.ws[L.OP_DOUBLE_BACKWARD])

    def step(self, src=None, outs=None):
        self.transpose(src)
        self.fwd(src, outs)
        self.bwd(src, outs)
        self.dbl(src, outs)


def time_ms(fn, steps, flush):
    """Mean device time (CUDA events on the current stream) of fn over `steps`
    calls, L2 flushed (a buffer of twice its size zeroed) before each, outside
    the events."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in evs:
        flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


def e2e_pipelined(work, host, hout, steps):
    """Mean time per step of `steps` steps that each copy their inputs in
    (pinned host -> device), run the step and copy every output back (device ->
    pinned host), with copies on their own streams: step i's inputs arrive
    while step i-1 computes, and its outputs leave while step i+1 computes
    (inputs and outputs double-buffered).  One event pair around the whole
    sequence, on the compute stream, after every copy has been joined."""
    import torch
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ins = [work.d, {k: torch.empty_like(v) for k, v in work.d.items()}]
    outs = [work.outs, {k: torch.empty_like(v) for k, v in work.outs.items()}]
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]      # inputs of buffer j landed
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]    # the step that read buffer j finished
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]     # outputs of buffer j copied out
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(comp)

    def copy_in(j):
        s_in.wait_event(t0)
        s_in.wait_event(ev_used[j])
        with torch.cuda.stream(s_in):
            for k, v in host.items():
                ins[j][k].copy_(v, non_blocking=True)
        ev_in[j].record(s_in)

    for j in range(2):
        ev_used[j].record(comp)
        ev_out[j].record(comp)
    copy_in(0)
    for i in range(steps):
        j = i & 1
        if i + 1 < steps:
            copy_in(1 - j)
        comp.wait_event(ev_in[j])
        comp.wait_event(ev_out[j])  # the copy-out of step i-2 from this buffer is done
        work.step(ins[j], outs[j])
        ev_used[j].record(comp)
        s_out.wait_event(ev_used[j])
        with torch.cuda.stream(s_out):
            for k, v in outs[j].items():
                hout[k].copy_(v, non_blocking=True)
        ev_out[j].record(s_out)
    comp.wait_event(ev_out[0])
    comp.wait_event(ev_out[1])
    comp.wait_stream(s_in)
    t1.record(comp)
    t1.synchronize()
    return t0.elapsed_time(t1) / steps


def per_direction(work, steps, flush):
    """edges/s of the forward alone, forward + backward (dx, dTheta, dvec; the
    sender-sorted view is built once per graph, outside), and the double
    backward alone (gg_x, gg_vec)."""
    work.transpose()
    t_f = time_ms(work.fwd, steps, flush)
    t_fb = time_ms(lambda: (work.fwd(), work.bwd()), steps, flush)
    t_d = time_ms(work.dbl, steps, flush)
    E = work.E
    return {"fwd_edges_per_s": E / (t_f * 1e-3), "fwd_bwd_edges_per_s": E / (t_fb * 1e-3),
            "dbl_edges_per_s": E / (t_d * 1e-3), "fwd_ms": t_f, "fwd_bwd_ms": t_fb, "dbl_ms": t_d}


def roofline(T, plan, prof_ms, E, workload_key):
    """FP32-ALU roofline of the dominant phase (algorithmic FMAs, see work_model).
    `traffic` comes from the ncu record of that phase only when the record was
    taken on this workload (config, family, gemm) and on the current sources."""
    peaks, peak_src = measured_peaks()
    wm = work_model(T, plan)
    dom = max(prof_ms, key=lambda k: prof_ms[k])
    roof = {"phase": dom, "bound": None, "achieved": None, "peak": None, "unit": None, "frac": None,
            "traffic": None}
    sm_max = peaks.get("sm_max_mhz", 1965.0)
    if dom in wm:
        flops = 2.0 * wm[dom] * E
        ach = flops / (prof_ms[dom] * 1e-3) / 1e12
        peak = N_SM * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
        roof.update(bound="alu", achieved=ach, peak=peak, unit="TFLOP/s", frac=ach / peak,
                    peak_source=f"148 SM x 128 FP32 lanes x 2 x {sm_max:.0f} MHz (max SM clock, {peak_src} peaks)",
                    work=f"{wm[dom]} algorithmic FMA per edge x {E} edges")
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            tr = json.load(f).get(dom)
        if tr and tr.get("workload") == workload_key and tr.get("sources_sha256") == sources_digest(tr["sources"]):
            roof["traffic"] = tr["dram_bytes_per_launch"]
            roof["traffic_kernel"] = tr["kernel"]
    except (OSError, ValueError):
        pass
    return roof


SUITE = {
    # entry: (config, degree, gemm)
    "tiny": ("tiny", None, "fp32"),
    "mace": ("mace", None, "fp32"),
    "sweep25": ("sweep", 25, "fp32"),
    "sweep100": ("sweep", 100, "fp32"),
    "sweep400": ("sweep", 400, "fp32"),
    "wide_fp32": ("wide", None, "fp32"),
    "wide_tf32": ("wide", None, "tf32"),
    "capacity": ("capacity", None, "fp32"),
}


def run_suite(args):
    """One JSON line per workload: edges/s of fwd, fwd+bwd and the double
    backward, peak allocated memory (total and workspace), and the FP32-ALU
    roofline fraction of the dominant edge-stream kernel of the full step."""
    import torch

    import equivariant_gnn_tensor_receiver_b200 as T
    from equivariant_gnn_tensor_receiver_b200 import _lib as L
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for name in args.suite_configs.split(","):
        cfg, degree, gemm = SUITE[name]
        cap = 8 << 30 if cfg == "capacity" else 0
        steps = 2 if cfg == "capacity" else args.steps
        graph = W.graph_for(cfg, 0, degree)
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        w = Work(T, L, cfg, graph, gemm, args.family, cap, dev)
        for _ in range(max(1, min(args.warmup, 3))):
            w.step()
        torch.cuda.synchronize()
        L.tpconv_profile_reset()
        L.tpconv_profile_enable(True)
        t_step = time_ms(w.step, steps, flush)
        L.tpconv_profile_enable(False)
        prof_ms = {k: ms / steps for k, (ms, _) in L.profile_all().items()}
        pd = per_direction(w, steps, flush)
        peak = torch.cuda.max_memory_allocated(dev) - base
        inputs = sum(v.numel() * v.element_size() for v in w.d.values())
        outputs = sum(v.numel() * v.element_size() for v in w.outs.values())
        line = {"suite": name, "workload": WORKLOADS[cfg].format(d=degree or 25), "gemm": gemm,
                "family": args.family, "nodes": w.N, "edges": w.E, "steps": steps,
                **{k: v for k, v in pd.items()},
                "step_edges_per_s": w.E / (t_step * 1e-3), "step_ms": t_step,
                "peak_mem_bytes": peak, "workspace_bytes": w.ws_bytes, "inputs_bytes": inputs,
                "outputs_bytes": outputs,
                "roofline": roofline(T, w.plan, prof_ms, w.E, f"{cfg}/{args.family}/{gemm}"),
                "phases_ms": {k: round(v, 4) for k, v in prof_ms.items() if v > 0}}
        print(json.dumps(line), flush=True)
        del w
        torch.cuda.synchronize()


def run_sharded(args):
    """One graph (seed 0) over all ranks by receiver ranges: every step runs
    forward, backward and double backward through the sharded operator,
    collectives included (strong scaling).  Time = max over ranks."""
    import datetime

    import torch
    import torch.distributed as dist

    import equivariant_gnn_tensor_receiver_b200 as T
    from equivariant_gnn_tensor_receiver_b200.sharded import LibraryOps, ShardedConv
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    c = W.CONFIGS[args.config]
    rowptr, col, vec = W.graph_for(args.config, 0, args.degree)
    N, E = len(rowptr) - 1, len(col)
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"], gemm=args.gemm, family=args.family)
    sc = ShardedConv(rowptr, col, rank, world, None, device=dev)
    lg = sc.local
    f32 = torch.float32
    todev = lambda a: torch.as_tensor(np.ascontiguousarray(a), dtype=f32, device=dev)
    sc.ops = LibraryOps(plan, todev(vec[lg.edges]))
    lo, hi = lg.lo, lg.hi
    x = todev(W.normal((N, plan.dim_in), 10)[lo:hi])
    th = todev(W.theta(theta_segments(plan.paths, plan.R, args.family), 11))
    g = todev(W.normal((N, plan.dim_out), 12)[lo:hi])
    ggx = todev(W.normal((N, plan.dim_in), 13)[lo:hi])
    ggv = todev(W.normal((E, 3), 14)[lg.edges])
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step():
        sc.forward(x, th)
        sc.backward(x, th, g)
        sc.double_backward(x, th, g, ggx, ggv, None)

    barrier = (lambda: dist.barrier()) if world > 1 else (lambda: None)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    barrier()
    ms = time_ms(step, args.steps, flush)
    ms_max = reduce_over_ranks(ms, "max", world, dev)
    if rank == 0:
        line = {"metric": METRIC, "value": E / (ms_max * 1e-3), "unit": "edges/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_max, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": workload(args), "nodes": N, "edges": E, "gemm": args.gemm,
                           "family": args.family,
                           "step": "fwd + bwd(dx,dTheta,dvec) + double bwd(gg_x,gg_vec), sharded",
                           "l2": "256 MiB buffer zeroed before every timed step, outside the events",
                           "parallelism": f"receiver ranges over {world} ranks: all-gather x, reduce-scatter "
                                          "dx / d_x, all-reduce dTheta / d_Theta (NCCL)"}}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_ours(args):
    import torch

    import equivariant_gnn_tensor_receiver_b200 as T
    from equivariant_gnn_tensor_receiver_b200 import _lib as L

    rank, world, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    graph = W.graph_for(args.config, rank, args.degree)
    rowptr, col, vec = graph
    N, E = len(rowptr) - 1, len(col)
    cap = args.workspace_cap if args.workspace_cap is not None else (8 << 30 if args.config == "capacity" else 0)
    work = Work(T, L, args.config, graph, args.gemm, args.family, cap, dev, seed=rank)
    plan, host, d, outs, ws_bytes = work.plan, work.host, work.d, work.outs, work.ws_bytes
    hout = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in outs.items()}
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    step = work.step

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    allmax = lambda v: reduce_over_ranks(v, "max", world, dev)
    allsum = lambda v: reduce_over_ranks(v, "sum", world, dev)

    for _ in range(max(args.warmup, 3)):
        step(d)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base_alloc = torch.cuda.memory_allocated(dev)
    L.tpconv_profile_reset()
    L.tpconv_profile_enable(True)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clk_path = args.clock_log.format(rank=rank) if args.clock_log else os.path.join(
        tempfile.gettempdir(), f"tpconv_clocks_{os.getpid()}_{rank}.csv")
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index, clk_path) as clk:
        time.sleep(0.3)
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record()
            step(d)
            evs[i][1].record()
        torch.cuda.synchronize()
    barrier()
    L.tpconv_profile_enable(False)
    step_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    job_value, step_ms_max, E_total = job_throughput(E, step_ms, world, dev)
    peak_mem = torch.cuda.max_memory_allocated(dev)
    prof = L.profile_all()
    launches = int(sum(n for _, n in prof.values()))

    # end to end: every step copies its inputs from pinned host memory and all
    # its outputs back to pinned host memory, inside the timed region
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in outs.values())
    barrier()
    e2e_ms = allmax(e2e_pipelined(work, host, hout, args.steps))

    # roofline of the dominant phase
    phase_ms = {k: ms / args.steps for k, (ms, _) in prof.items()}
    roof = roofline(T, plan, phase_ms, E, f"{args.config}/{args.family}/{args.gemm}")

    per_dir = per_direction(work, args.steps, flush)
    for k in ("fwd_ms", "fwd_bwd_ms", "dbl_ms"):  # slowest rank; every rank takes the same steps
        per_dir[k] = allmax(per_dir[k])
    E_all = allsum(float(E))
    per_dir.update(fwd_edges_per_s=E_all / (per_dir["fwd_ms"] * 1e-3),
                   fwd_bwd_edges_per_s=E_all / (per_dir["fwd_bwd_ms"] * 1e-3),
                   dbl_edges_per_s=E_all / (per_dir["dbl_ms"] * 1e-3))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        procs = args.oracle_procs or min(32, host_cores())
        r = parallel_oracle(args.config, args.family, procs, 4, 1, 2)
        cpu = {k: r[k] for k in ("value", "unit", "cores", "kind", "sample")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": job_value, "unit": "edges/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": workload(args), "workspace_cap": cap, "nodes_per_gpu": N, "edges_per_gpu": E, "gemm": args.gemm,
                       "family": args.family,
                       "step": "graph transpose + fwd + bwd(dx,dTheta,dvec) + double bwd(gg_x,gg_vec)",
                       "l2": "256 MiB buffer zeroed before every timed step, outside the events",
                       "parallelism": f"{world} independent replicas (one graph per rank)"},
            "e2e": {"value": E_total / (e2e_ms * 1e-3), "unit": "edges/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "copies": "each step's inputs in and outputs out, on copy streams overlapping the "
                              "neighbouring steps' compute (double-buffered); no L2 flush (the copies "
                              "rewrite the inputs every step; workspaces exceed L2)"},
            "gpu_launches": launches,
            "roofline": roof,
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "per_direction": per_dir,
            "phases_ms": {k: round(v, 4) for k, v in phase_ms.items() if v > 0},
            "peak_mem_bytes": peak_mem, "workspace_bytes": ws_bytes, "resident_bytes_before_step": base_alloc,
            "library_static_bytes": L.static_device_bytes(),
        }
        print(json.dumps(line), flush=True)
    if args.parity_sample and world == 1:
        work.step()  # outputs of one step over the resident inputs
        torch.cuda.synchronize()
        procs = args.oracle_procs or min(32, host_cores())
        print(json.dumps(parity_check(args, work, graph, procs, args.parity_sample)), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.suite:
        run_suite(args)
    elif args.shard:
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
