"""Host logic of the benchmark's sampled parity check (no GPU): the oracle on
the sub-problem that the check builds for sampled receivers, senders and edges
reproduces the oracle on the whole graph for exactly those rows."""

import importlib.util
import os
import sys

import numpy as np

import workloads as W
from oracle import conv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    if "bench" in sys.modules:
        return sys.modules["bench"]
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    sys.modules["bench"] = m  # its pool workers are pickled by module name
    spec.loader.exec_module(m)
    return m


def test_sub_problems_reproduce_the_whole_graph():
    B = _bench()
    c = W.CONFIGS["tiny"]
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"], c["radial_params"])
    rowptr, col, vec = W.graph_for("tiny", 2)
    N, E = len(rowptr) - 1, len(col)
    x, g = W.normal((N, prob.dim_in), 1), W.normal((N, prob.dim_out), 2)
    th = W.theta([(c["R"] * p.c_in * p.c_out, 0.2) for p in prob.paths], 3)
    ggx, ggv = W.normal((N, prob.dim_in), 4), W.normal((E, 3), 5)
    full_f = conv.forward(prob, rowptr, col, vec, x, th)
    full_b = conv.backward(prob, rowptr, col, vec, x, th, g)
    full_d = conv.double_backward(prob, rowptr, col, vec, x, th, g, ggx, ggv, None)
    rp = np.asarray(rowptr, dtype=np.int64)
    rs = np.array([3, 17, 40])
    edges = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in rs])
    lrp, lc, eids, recvs, nodes = B._sub_problem(rowptr, col, edges)
    assert np.array_equal(np.sort(eids), np.sort(edges)) and np.array_equal(recvs, rs)
    pos = {int(v): i for i, v in enumerate(nodes)}
    rows = [pos[int(r)] for r in rs]
    a = {"rowptr": lrp, "col": lc, "vec": vec[eids], "x": x[nodes], "theta": th, "g": g[nodes],
         "gg_x": ggx[nodes], "gg_vec": ggv[eids]}
    out = B._parity_worker(("recv", "tiny", "full", a))["out"]
    assert np.allclose(out[rows], full_f[rs], rtol=0, atol=1e-12)
    d_g = B._parity_worker(("recv_dbl", "tiny", "full", a))["d_g"]
    assert np.allclose(d_g[rows], full_d["d_g"][rs], rtol=0, atol=1e-11)
    # senders: all their out-edges
    ss = np.array([5, 30])
    es = np.nonzero(np.isin(col, ss))[0]
    lrp, lc, eids, recvs, nodes = B._sub_problem(rowptr, col, es)
    pos = {int(v): i for i, v in enumerate(nodes)}
    a = {"rowptr": lrp, "col": lc, "vec": vec[eids], "x": x[nodes], "theta": th, "g": g[nodes],
         "gg_x": ggx[nodes], "gg_vec": ggv[eids]}
    rows = [pos[int(s)] for s in ss]
    assert np.allclose(B._parity_worker(("send", "tiny", "full", a))["dx"][rows], full_b["dx"][ss], atol=1e-11)
    assert np.allclose(B._parity_worker(("send_dbl", "tiny", "full", a))["d_x"][rows], full_d["d_x"][ss],
                       atol=1e-10)
    # single edges
    ee = np.array([0, 77, 300, 511])
    lrp, lc, eids, recvs, nodes = B._sub_problem(rowptr, col, ee)
    a = {"rowptr": lrp, "col": lc, "vec": vec[eids], "x": x[nodes], "theta": th, "g": g[nodes],
         "gg_x": ggx[nodes], "gg_vec": ggv[eids]}
    r = B._parity_worker(("edge", "tiny", "full", a))
    order = np.argsort(eids)
    assert np.allclose(r["dvec"][order], full_b["dvec"][np.sort(eids)], atol=1e-11)
    assert np.allclose(r["d_vec"][order], full_d["d_vec"][np.sort(eids)], atol=1e-10)


def test_sampled_parity_end_to_end_with_isolated_nodes():
    """The whole sampling path (job building, worker pool, row assembly) with
    the oracle's own full-graph results as the 'device' outputs: every error is
    at rounding level.  The graph has isolated nodes (no in- or out-edges) and
    more edges than nodes, so node rows and edge rows must not be confused."""
    B = _bench()
    c = W.CONFIGS["tiny"]
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"], c["radial_params"])
    rowptr, col, vec = W.graph_for("tiny", 3)
    N0 = len(rowptr) - 1
    # append 6 isolated nodes
    rowptr = np.concatenate([rowptr, np.full(6, rowptr[-1], dtype=rowptr.dtype)])
    N, E = len(rowptr) - 1, len(col)
    assert E > N
    f32 = lambda a: np.asarray(a, dtype=np.float32)
    inputs = {"x": f32(W.normal((N, prob.dim_in), 1)), "g": f32(W.normal((N, prob.dim_out), 2)),
              "theta": f32(W.theta([(c["R"] * p.c_in * p.c_out, 0.2) for p in prob.paths], 3)),
              "gg_x": f32(W.normal((N, prob.dim_in), 4)), "gg_vec": f32(W.normal((E, 3), 5)), "vec": f32(vec)}
    d = {k: np.asarray(v, dtype=np.float64) for k, v in inputs.items()}
    full = {"out": conv.forward(prob, rowptr, col, d["vec"], d["x"], d["theta"])}
    rb = conv.backward(prob, rowptr, col, d["vec"], d["x"], d["theta"], d["g"])
    rd = conv.double_backward(prob, rowptr, col, d["vec"], d["x"], d["theta"], d["g"], d["gg_x"], d["gg_vec"], None)
    full.update(dx=rb["dx"], dvec=rb["dvec"], d_g=rd["d_g"], d_x=rd["d_x"], d_vec=rd["d_vec"])
    assert np.abs(full["out"][N0:]).max() == 0
    errs, sampled = B.sampled_parity("tiny", "full", (rowptr, col, vec), inputs,
                                     lambda key, idx: full[key][np.asarray(idx)], 2, N)
    assert sampled["receivers"] == N  # every node sampled, isolated ones included
    assert set(errs) == {"out", "d_g", "dx", "d_x", "dvec", "d_vec"}
    assert max(errs.values()) < 1e-12, errs


def test_traffic_record_applies_only_to_its_workload():
    """The ncu DRAM-traffic figure of the dominant phase is reported only for the
    workload (config / family / gemm) and the sources it was captured on."""
    import json
    B = _bench()
    import equivariant_gnn_tensor_receiver_b200 as T
    c = W.CONFIGS["mace"]
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"])
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)["dbl_edge_r"]
    prof = {"fwd_edge": 0.6, "dbl_edge_r": 2.2, "bwd_edge_r": 1.3}
    own = B.roofline(T, plan, prof, 213738, rec["workload"])
    other = B.roofline(T, plan, prof, 213738, "wide/full/fp32")
    assert own["phase"] == other["phase"] == "dbl_edge_r"
    if rec["sources_sha256"] == B.sources_digest(rec["sources"]):
        assert own["traffic"] == rec["dram_bytes_per_launch"] and own["traffic_kernel"] == rec["kernel"]
    else:  # the kernel changed since the capture: no traffic figure at all
        assert own["traffic"] is None
    assert other["traffic"] is None and "traffic_kernel" not in other
    assert own["frac"] == other["frac"] and 0 < own["frac"] < 1
