"""GPU parity at the workloads' own shapes: the wide operator (128 channels per
block up to l = 3), the edge-scaling sweep at its lowest and highest degree, and
the Theta gradients over every node of the mace-like and wide layers.

Each check compares the library (through the C ABI) with the fp64 oracle
element by element on quantities the oracle can compute exactly from a part of
the graph:
  * out and d_g of sampled receivers depend only on those receivers' edges;
  * dvec, d_vec of an edge depend only on the edge and its receiver;
  * dx, d_x of sampled senders depend only on their out-edges;
  * dTheta, d_Theta sum over every edge, so they are checked on a graph that
    keeps every node but only the edges of sampled receivers: the library still
    runs its node-level contractions over all N nodes (all K splits, all tiles),
    and the oracle computes the same sums exactly.

Tolerance: max-norm relative error <= 1e-5 for the fp32 path (3xTF32 or FFMA
Theta contractions), <= 5e-3 when the Theta contraction runs in TF32.
"""

import numpy as np
import pytest

import workloads as W
from oracle import conv

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "simt": 1e-5, "tf32": 5e-3}


@pytest.fixture(scope="module")
def T():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import equivariant_gnn_tensor_receiver_b200 as T
    T.lib()
    return T


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    d = np.abs(b).max()
    return np.abs(a - b).max() / (d if d > 0 else 1.0)


def dev(a, dtype=None):
    import torch
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype or torch.float32, device="cuda")


def r32(a):
    return np.asarray(a).astype(np.float32).astype(np.float64)


class Setup:
    """Plan, oracle problem and fp32-rounded seeded inputs of one workload."""

    def __init__(self, T, name, graph, gemm, seed):
        import torch
        c = W.CONFIGS[name]
        self.T = T
        self.plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                           radial_params=c["radial_params"], gemm=gemm)
        self.prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                                 tuple(c["radial_params"]))
        self.rowptr, self.col, vec = graph
        self.vec = r32(vec)
        self.N, self.E = len(self.rowptr) - 1, len(self.col)
        R = c["R"]
        self.x = r32(W.normal((self.N, self.prob.dim_in), seed + 1))
        self.th = r32(W.theta([(R * p.c_in * p.c_out, 1.0 / np.sqrt(R * p.c_in)) for p in self.prob.paths],
                              seed + 2))
        self.g = r32(W.normal((self.N, self.prob.dim_out), seed + 3))
        self.ggx = r32(W.normal((self.N, self.prob.dim_in), seed + 4))
        self.ggv = r32(W.normal((self.E, 3), seed + 5))
        self.ggt = r32(W.normal(self.th.shape, seed + 6) * 0.05)
        self.recv = np.repeat(np.arange(self.N), np.diff(self.rowptr))
        self.G = T.Graph(dev(self.rowptr, torch.int32), dev(self.col, torch.int32), dev(self.vec))

    def sub_csr(self, mask):
        """Receiver CSR over all N nodes that holds only the masked edges."""
        return np.concatenate([[0], np.cumsum(np.bincount(self.recv[mask], minlength=self.N))]).astype(np.int64)


def check_sampled(T, name, graph, gemm, seed, n_recv, n_send, dbl=True):
    """Forward, backward and (force-training shape) double backward of the full
    graph, checked on sampled receivers, their edges and sampled senders."""
    import torch
    S = Setup(T, name, graph, gemm, seed)
    tol = TOL[gemm]
    out = T.forward(S.plan, S.G, dev(S.x), dev(S.th)).double().cpu().numpy()
    bw = T.backward(S.plan, S.G, dev(S.x), dev(S.th), dev(S.g), want=("dx", "dvec"))
    bw = {k: v.double().cpu().numpy() for k, v in bw.items()}
    if dbl:
        o2 = T.double_backward(S.plan, S.G, dev(S.x), dev(S.th), dev(S.g), dev(S.ggx), dev(S.ggv), None)
        o2 = {k: v.double().cpu().numpy() for k, v in o2.items()}
    torch.cuda.synchronize()
    rs = np.random.default_rng(seed).choice(S.N, n_recv, replace=False)
    em = np.isin(S.recv, rs)
    sub = S.sub_csr(em)
    ref = conv.forward(S.prob, sub, S.col[em], S.vec[em], S.x, S.th)
    errs = {"out": rel(out[rs], ref[rs])}
    rb = conv.backward(S.prob, sub, S.col[em], S.vec[em], S.x, S.th, S.g)
    errs["dvec"] = rel(bw["dvec"][em], rb["dvec"])
    ss = np.random.default_rng(seed + 100).choice(S.N, n_send, replace=False)
    sm = np.isin(S.col, ss)
    sub_s = S.sub_csr(sm)
    rbs = conv.backward(S.prob, sub_s, S.col[sm], S.vec[sm], S.x, S.th, S.g)
    errs["dx"] = rel(bw["dx"][ss], rbs["dx"][ss])
    if dbl:
        r2 = conv.double_backward(S.prob, sub, S.col[em], S.vec[em], S.x, S.th, S.g, S.ggx, S.ggv[em], None)
        errs["d_g"] = rel(o2["d_g"][rs], r2["d_g"][rs])
        errs["d_vec"] = rel(o2["d_vec"][em], r2["d_vec"])
        r2s = conv.double_backward(S.prob, sub_s, S.col[sm], S.vec[sm], S.x, S.th, S.g, S.ggx, S.ggv[sm], None)
        errs["d_x"] = rel(o2["d_x"][ss], r2s["d_x"][ss])
    bad = {k: v for k, v in errs.items() if not v < tol}
    assert not bad, (name, gemm, errs)
    return errs


@pytest.mark.parametrize("gemm", ["fp32", "tf32"])
def test_wide_operator_sampled(T, gemm):
    """The wide operator: 8192 nodes, mean degree 32, 128x0e+128x1o+128x2e+128x3o
    in and out, SH l <= 3, R = 8 Bessel (23 paths, l = 3 features on both sides,
    128 channels per block)."""
    check_sampled(T, "wide", W.graph_for("wide", 0), gemm, seed=81, n_recv=10, n_send=8)


@pytest.mark.parametrize("degree", [25, 400])
def test_sweep_sampled(T, degree):
    """The edge-scaling sweep at both ends: 20000 nodes, mean degree 25
    (0.5 M edges) and 400 (8 M edges), 32x0e+32x1o+32x2e, SH l <= 2, R = 8."""
    check_sampled(T, "sweep", W.graph_for("sweep", 0, degree), "fp32", seed=91, n_recv=12, n_send=8)


@pytest.mark.parametrize("name,gemm,n_recv", [("mace", "fp32", 64), ("mace", "tf32", 64), ("wide", "fp32", 24)])
def test_theta_gradients_over_all_nodes(T, name, gemm, n_recv):
    """dTheta (backward) and d_Theta (double backward, with and without
    gg_Theta) element by element over every node of the layer: the graph keeps
    all N nodes but only the edges of n_recv sampled receivers, so the node-level
    Theta contractions run over the full node range while the oracle sums
    exactly the same edges."""
    import torch
    full = W.graph_for(name, 0)
    rowptr, col, vec = full
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    rs = np.random.default_rng(7).choice(N, n_recv, replace=False)
    em = np.isin(recv, rs)
    sub = np.concatenate([[0], np.cumsum(np.bincount(recv[em], minlength=N))]).astype(np.int32)
    S = Setup(T, name, (sub, col[em], vec[em]), gemm, seed=101)
    tol = TOL[gemm]
    dth = T.backward(S.plan, S.G, dev(S.x), dev(S.th), dev(S.g), want=("dtheta",))["dtheta"]
    o_no_t = T.double_backward(S.plan, S.G, dev(S.x), dev(S.th), dev(S.g), dev(S.ggx), dev(S.ggv), None,
                               want=("d_theta", "d_x"))
    o_t = T.double_backward(S.plan, S.G, dev(S.x), dev(S.th), dev(S.g), dev(S.ggx), dev(S.ggv), dev(S.ggt),
                            want=("d_theta", "d_x"))
    torch.cuda.synchronize()
    rb = conv.backward(S.prob, S.rowptr, S.col, S.vec, S.x, S.th, S.g)
    assert rel(dth.double().cpu().numpy(), rb["dtheta"]) < tol
    r2 = conv.double_backward(S.prob, S.rowptr, S.col, S.vec, S.x, S.th, S.g, S.ggx, S.ggv, None)
    assert rel(o_no_t["d_theta"].double().cpu().numpy(), r2["d_theta"]) < tol
    assert rel(o_no_t["d_x"].double().cpu().numpy(), r2["d_x"]) < tol
    r3 = conv.double_backward(S.prob, S.rowptr, S.col, S.vec, S.x, S.th, S.g, S.ggx, S.ggv, S.ggt)
    assert rel(o_t["d_theta"].double().cpu().numpy(), r3["d_theta"]) < tol
    assert rel(o_t["d_x"].double().cpu().numpy(), r3["d_x"]) < tol
