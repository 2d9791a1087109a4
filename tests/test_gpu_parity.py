"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Tolerance: max-norm relative error ||gpu - ref||_inf / ||ref||_inf <= 1e-5 for
the fp32 path (the operator's stated bar for fp32 arithmetic); 5e-3 when the
Theta contraction runs with TF32 operands.
"""

import numpy as np
import pytest

import workloads as W
from oracle import conv

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-5
TOL_LOWP = 5e-3
TOL = {"simt": TOL_FP32, "fp32": TOL_FP32, "tf32": TOL_LOWP}


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


def dev(a, dtype):
    import torch
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype, device="cuda")


def make(T, irr_in, lsh, irr_out, R, radial, rp, graph, seed, gemm="simt", cap=0):
    import torch
    rowptr, col, vec = graph
    plan = T.Plan(irr_in, lsh, irr_out, R, radial=radial, radial_params=rp, gemm=gemm, workspace_cap=cap)
    prob = conv.Problem(irr_in, lsh, irr_out, R, radial, rp)
    N = len(rowptr) - 1
    x = W.normal((N, prob.dim_in), seed + 1)
    th = W.theta([(R * p.c_in * p.c_out, 1.0 / np.sqrt(R * p.c_in)) for p in prob.paths], seed + 2)
    g = W.normal((N, prob.dim_out), seed + 3)
    G = T.Graph(dev(rowptr, torch.int32), dev(col, torch.int32), dev(vec, torch.float32))
    # the oracle sees exactly the fp32-rounded inputs the GPU sees
    x32, th32, g32 = (a.astype(np.float32).astype(np.float64) for a in (x, th, g))
    vec32 = vec.astype(np.float32).astype(np.float64)
    return plan, prob, G, (rowptr, col, vec32, x32, th32, g32)


def run_fwd_bwd(T, plan, G, inp):
    import torch
    rowptr, col, vec, x, th, g = inp
    xd, thd, gd = dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32)
    out = T.forward(plan, G, xd, thd)
    bw = T.backward(plan, G, xd, thd, gd, want=("dx", "dtheta", "dvec", "dY", "db"))
    torch.cuda.synchronize()
    return out.cpu().numpy(), {k: v.cpu().numpy() for k, v in bw.items()}


CASES = {
    # name: (irreps_in, lsh, irreps_out, R, radial, params, graph)
    "tiny": ("8x0e+8x1o", 2, "8x0e+8x1o", 4, "gaussian", (0.5, 5.0), lambda: W.graph_for("tiny", 0)),
    "mixed_l3": ("5x0e+3x1o+2x1e+4x2e+3x3o", 3, "3x0e+2x0o+4x1o+1x1e+3x2e+2x3o+1x3e", 3, "bessel", (5.0,),
                 lambda: W.random_graph(40, 400, 5, r_min=0.6, r_max=4.8)),
    "wide_channels": ("40x0e+36x1o", 1, "33x0e+70x1o", 8, "bessel", (5.0,),
                      lambda: W.random_graph(30, 250, 6, r_min=0.6, r_max=4.8)),
    "radius_small": ("16x0e+16x1o+16x2e", 3, "16x0e+16x1o+16x2e", 8, "bessel", (5.0,),
                     lambda: W.radius_graph(300, 14.0, 5.0, 7)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_forward_backward_parity(T, case):
    irr_in, lsh, irr_out, R, rad, rp, gf = CASES[case]
    plan, prob, G, inp = make(T, irr_in, lsh, irr_out, R, rad, rp, gf(), seed=11)
    rowptr, col, vec, x, th, g = inp
    out, bw = run_fwd_bwd(T, plan, G, inp)
    ref = conv.forward(prob, rowptr, col, vec, x, th)
    assert rel(out, ref) < TOL_FP32
    rb = conv.backward(prob, rowptr, col, vec, x, th, g)
    for k in ("dx", "dtheta", "dvec", "dY", "db"):
        assert rel(bw[k], rb[k]) < TOL_FP32, (k, rel(bw[k], rb[k]))


def test_edge_cases_empty_and_hub(T):
    # receivers with no edges, one hub receiver of degree 300 (many batches),
    # one sender with many out-edges, and a chunked workspace
    g = W.rng(3)
    N = 50
    recv = np.concatenate([np.full(300, 7), g.integers(20, 30, size=100)])
    send = np.concatenate([g.integers(0, N, size=300), np.full(100, 41)])
    d = g.normal(size=(400, 3))
    vec = d / np.linalg.norm(d, axis=1, keepdims=True) * g.uniform(0.6, 4.8, size=(400, 1))
    graph = W._to_csr(N, send, recv, vec)
    for cap in (0, 40_000):
        plan, prob, G, inp = make(T, "6x0e+5x1o+3x2e", 2, "4x0e+6x1o+2x2e", 5, "bessel", (5.0,), graph, seed=21,
                                  cap=cap)
        rowptr, col, vec32, x, th, gg = inp
        out, bw = run_fwd_bwd(T, plan, G, inp)
        ref = conv.forward(prob, rowptr, col, vec32, x, th)
        assert rel(out, ref) < TOL_FP32
        assert np.all(out[:7] == 0) and np.all(out[8:20] == 0)
        rb = conv.backward(prob, rowptr, col, vec32, x, th, gg)
        for k in ("dx", "dtheta", "dvec"):
            assert rel(bw[k], rb[k]) < TOL_FP32, (cap, k)


def test_power_law_hubs_split_into_pieces(T):
    """Heavy-tailed degrees: three hub receivers (1500, 900, 600 in-edges) and
    two hub senders (1200 out-edges each) over a sparse background.  Segments
    longer than max(256, 4 x mean degree) edges run as several pieces that add
    into zeroed state rows, and the receivers' batches are spread over warps;
    forward, backward and double backward against the oracle."""
    import torch
    g = W.rng(17)
    N = 400
    bg_r, bg_s = g.integers(0, N, size=3200), g.integers(0, N, size=3200)
    recv = np.concatenate([np.full(1500, 11), np.full(900, 203), np.full(600, 390), bg_r,
                           g.integers(0, N, size=2400)])
    send = np.concatenate([g.integers(0, N, size=3000), bg_s, np.full(1200, 77), np.full(1200, 298)])
    E = len(recv)
    dvec = g.normal(size=(E, 3))
    vec = dvec / np.linalg.norm(dvec, axis=1, keepdims=True) * g.uniform(0.6, 4.8, size=(E, 1))
    graph = W._to_csr(N, send, recv, vec)
    irr_in, irr_out = "8x0e+8x1o+4x2e", "8x0e+4x1o+8x2e"
    plan, prob, G, inp = make(T, irr_in, 2, irr_out, 8, "bessel", (5.0,), graph, seed=23)
    rowptr, col, vec32, x, th, gg = inp
    assert np.diff(rowptr).max() > 4 * 256 and np.bincount(col).max() >= 1200
    out, bw = run_fwd_bwd(T, plan, G, inp)
    assert rel(out, conv.forward(prob, rowptr, col, vec32, x, th)) < TOL_FP32
    rb = conv.backward(prob, rowptr, col, vec32, x, th, gg)
    for k in ("dx", "dtheta", "dvec"):
        assert rel(bw[k], rb[k]) < TOL_FP32, k
    r32 = lambda a: a.astype(np.float32).astype(np.float64)
    ggx, ggv = r32(W.normal(x.shape, 24)), r32(W.normal(vec32.shape, 25))
    ggt = r32(W.normal(th.shape, 26) * 0.05)
    o2 = T.double_backward(plan, G, dev(x, torch.float32), dev(th, torch.float32), dev(gg, torch.float32),
                           dev(ggx, torch.float32), dev(ggv, torch.float32), dev(ggt, torch.float32))
    torch.cuda.synchronize()
    ref2 = conv.double_backward(prob, rowptr, col, vec32, x, th, gg, ggx, ggv, ggt)
    for k in ("d_g", "d_x", "d_vec", "d_theta"):
        assert rel(o2[k].cpu().numpy(), ref2[k]) < TOL_FP32, k


def test_no_edges(T):
    import torch
    graph = (np.zeros(11, dtype=np.int32), np.zeros(0, dtype=np.int32), np.zeros((0, 3)))
    plan, prob, G, inp = make(T, "4x0e+2x1o", 1, "3x0e+2x1o", 4, "bessel", (5.0,), graph, seed=31)
    out, bw = run_fwd_bwd(T, plan, G, inp)
    assert np.all(out == 0) and np.all(bw["dx"] == 0) and np.all(bw["dtheta"] == 0)
    assert bw["dvec"].shape == (0, 3)


def test_graph_transpose_exact(T):
    import torch
    rowptr, col, vec = W.graph_for("mace", 0)
    plan = T.Plan("1x0e", 0, "1x0e", 1)
    G = T.Graph(dev(rowptr, torch.int32), dev(col, torch.int32), dev(vec, torch.float32))
    perm, s_rowptr, s_recv = (a.cpu().numpy() for a in G.transposed(plan))
    N, E = len(rowptr) - 1, len(col)
    order = np.lexsort((np.arange(E), col))
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    assert np.array_equal(perm[:E], order)
    assert np.array_equal(s_recv[:E], recv[order])
    assert np.array_equal(s_rowptr, np.concatenate([[0], np.cumsum(np.bincount(col, minlength=N))]))


@pytest.mark.parametrize("gemm", ["fp32", "tf32", "simt"])
def test_mace_full_size_sampled(T, gemm):
    """The mace layer at full size (4096 atoms, ~214k edges), forward and the
    per-edge / per-sender adjoints checked on sampled receivers, edges and
    senders, each of which the oracle computes exactly from its own edges.
    gemm selects the node-level Theta contraction: 3xTF32 or TF32 tensor cores
    (tcgen05) or FFMA."""
    import torch
    c = W.CONFIGS["mace"]
    graph = W.graph_for("mace", 0)
    plan, prob, G, inp = make(T, c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                              c["radial_params"], graph, seed=41, gemm=gemm)
    rowptr, col, vec, x, th, g = inp
    out, bw = run_fwd_bwd(T, plan, G, inp)
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    rs = np.random.default_rng(0).choice(N, 24, replace=False)
    em = np.isin(recv, rs)
    loc = {r: i for i, r in enumerate(rs)}
    Y, b, JY, Jb = conv.geometry(prob, vec[em], order=1)
    ref = conv.forward_core(prob, len(rs), col[em].astype(np.int64), np.array([loc[r] for r in recv[em]]), x, Y,
                            b, th)
    assert rel(out[rs], ref) < TOL[gemm], rel(out[rs], ref)
    # per-edge adjoints of the sampled receivers' edges (local quantities)
    gl = g[rs]
    _, _, dY, db = conv.backward_core(prob, len(rs), col[em].astype(np.int64),
                                      np.array([loc[r] for r in recv[em]]), x, Y, b, th, gl)
    dvec = np.einsum('em,emi->ei', dY, JY) + np.einsum('ek,eki->ei', db, Jb)
    assert rel(bw["dvec"][em], dvec) < TOL[gemm]
    # dx of sampled senders (all their out-edges)
    ss = np.random.default_rng(1).choice(N, 16, replace=False)
    sm = np.isin(col, ss)
    Y2, b2 = conv.geometry(prob, vec[sm])
    dx, _, _, _ = conv.backward_core(prob, N, col[sm].astype(np.int64), recv[sm], x, Y2, b2, th, g)
    assert rel(bw["dx"][ss], dx[ss]) < TOL[gemm]


def _sub_csr(N, recv, mask):
    """Receiver CSR over all N nodes holding only the masked edges (still receiver-sorted)."""
    return np.concatenate([[0], np.cumsum(np.bincount(recv[mask], minlength=N))]).astype(np.int64)


def _identity_ok(lhs_terms, rhs_terms):
    """Scalar identity sum(lhs) = sum(rhs) of fp32 results: the fp32 bar (1e-5)
    applied to the sums of absolute terms, the scale the rounding of every term
    contributes to (the sums themselves cancel by orders of magnitude)."""
    lhs = sum(float(t.sum()) for t in lhs_terms)
    rhs = sum(float(t.sum()) for t in rhs_terms)
    scale = sum(float(np.abs(t).sum()) for t in lhs_terms) + sum(float(np.abs(t).sum()) for t in rhs_terms)
    return abs(lhs - rhs) <= TOL_FP32 * scale, (lhs, rhs, scale)


@pytest.mark.parametrize("gemm", ["fp32"])
def test_mace_full_size_dtheta_identity(T, gemm):
    """dTheta at full size: out is linear in Theta, so <dTheta, D> = <g, out(x, D)>
    for any direction D (both sides from the library; dTheta sums over all edges,
    which the oracle cannot sample)."""
    import torch
    c = W.CONFIGS["mace"]
    plan, prob, G, inp = make(T, c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                              c["radial_params"], W.graph_for("mace", 0), seed=43, gemm=gemm)
    rowptr, col, vec, x, th, g = inp
    xd, thd, gd = dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32)
    dth = T.backward(plan, G, xd, thd, gd, want=("dtheta",))["dtheta"].double().cpu().numpy()
    D = W.normal(th.shape, 44).astype(np.float32)
    outD = T.forward(plan, G, xd, dev(D, torch.float32)).double().cpu().numpy()
    ok, info = _identity_ok([dth * D.astype(np.float64)], [g * outD])
    assert ok, info


def test_mace_full_size_double_backward_sampled(T):
    """The double backward of the bench step at full size (gg_x and gg_vec, no
    gg_Theta; 3xTF32 Theta contractions).  d_g of sampled receivers and d_vec of
    their edges depend only on those receivers' edges, d_x of sampled senders
    only on their out-edges: the oracle computes them exactly on those sub-graphs.
    d_Theta is checked through Psi's linearity in Theta:
    <d_Theta, D> = <gg_x, dx(D)> + <gg_vec, dvec(D)>."""
    import torch
    c = W.CONFIGS["mace"]
    plan, prob, G, inp = make(T, c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                              c["radial_params"], W.graph_for("mace", 0), seed=45, gemm="fp32")
    rowptr, col, vec, x, th, g = inp
    r32 = lambda a: a.astype(np.float32).astype(np.float64)
    ggx, ggv = r32(W.normal(x.shape, 46)), r32(W.normal(vec.shape, 47))
    xd, thd, gd = dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32)
    ggxd, ggvd = dev(ggx, torch.float32), dev(ggv, torch.float32)
    out = {k: v.double().cpu().numpy() for k, v in T.double_backward(plan, G, xd, thd, gd, ggxd, ggvd, None).items()}
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    rs = np.random.default_rng(2).choice(N, 20, replace=False)
    em = np.isin(recv, rs)
    ref = conv.double_backward(prob, _sub_csr(N, recv, em), col[em], vec[em], x, th, g, ggx, ggv[em], None)
    assert rel(out["d_g"][rs], ref["d_g"][rs]) < TOL_FP32
    assert rel(out["d_vec"][em], ref["d_vec"]) < TOL_FP32
    ss = np.random.default_rng(3).choice(N, 12, replace=False)
    sm = np.isin(col, ss)
    ref2 = conv.double_backward(prob, _sub_csr(N, recv, sm), col[sm], vec[sm], x, th, g, ggx, ggv[sm], None)
    assert rel(out["d_x"][ss], ref2["d_x"][ss]) < TOL_FP32
    D = W.normal(th.shape, 48).astype(np.float32)
    bw = T.backward(plan, G, xd, dev(D, torch.float32), gd, want=("dx", "dvec"))
    ok, info = _identity_ok([out["d_theta"] * D.astype(np.float64)],
                            [ggx * bw["dx"].double().cpu().numpy(), ggv * bw["dvec"].double().cpu().numpy()])
    assert ok, info


DBL_CASES = {
    "tiny_all": ("tiny", ("x", "v", "t")),
    "mixed_all": ("mixed_l3", ("x", "v", "t")),
    "mixed_force_shape": ("mixed_l3", ("x", "v")),
    "radius_only_vec": ("radius_small", ("v",)),
    "wide_only_theta_x": ("wide_channels", ("x", "t")),
}


@pytest.mark.parametrize("case", list(DBL_CASES))
def test_double_backward_parity(T, case):
    import torch
    base, which = DBL_CASES[case]
    irr_in, lsh, irr_out, R, rad, rp, gf = CASES[base]
    plan, prob, G, inp = make(T, irr_in, lsh, irr_out, R, rad, rp, gf(), seed=51)
    rowptr, col, vec, x, th, g = inp
    r32 = lambda a: a.astype(np.float32).astype(np.float64)
    ggx = r32(W.normal(x.shape, 52)) if "x" in which else None
    ggv = r32(W.normal(vec.shape, 53)) if "v" in which else None
    ggt = r32(W.normal(th.shape, 54) * 0.05) if "t" in which else None
    d = lambda a: None if a is None else dev(a, torch.float32)
    out = T.double_backward(plan, G, d(x), d(th), d(g), d(ggx), d(ggv), d(ggt))
    torch.cuda.synchronize()
    ref = conv.double_backward(prob, rowptr, col, vec, x, th, g, ggx, ggv, ggt)
    for k in ("d_g", "d_x", "d_vec", "d_theta"):
        got = out[k].cpu().numpy()
        if np.abs(ref[k]).max() == 0:
            assert np.abs(got).max() == 0, k
        else:
            assert rel(got, ref[k]) < TOL_FP32, (k, rel(got, ref[k]))


@pytest.mark.parametrize("gemm", ["fp32", "tf32"])
@pytest.mark.parametrize("irr", ["16x0e+16x1o+16x2e", "24x0e+40x1o"])
def test_tensor_core_mixing(T, gemm, irr):
    """Forward through the tcgen05 Theta contraction: M = nodes x (2l+1) with a
    ragged last 128-row tile, C_out below / between the 32..256 column tiles."""
    import torch
    graph = W.radius_graph(333, 15.0, 5.0, 8)
    plan, prob, G, inp = make(T, irr, 2, irr, 8, "bessel", (5.0,), graph, seed=61, gemm=gemm)
    rowptr, col, vec, x, th, g = inp
    out = T.forward(plan, G, dev(x, torch.float32), dev(th, torch.float32))
    torch.cuda.synchronize()
    ref = conv.forward(prob, rowptr, col, vec, x, th)
    assert rel(out.cpu().numpy(), ref) < TOL[gemm]
    dbl = T.double_backward(plan, G, dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32),
                            dev(W.normal(x.shape, 62), torch.float32), dev(W.normal(vec.shape, 63), torch.float32),
                            dev(W.normal(th.shape, 64) * 0.05, torch.float32), want=("d_g",))
    torch.cuda.synchronize()
    r32 = lambda a: a.astype(np.float32).astype(np.float64)
    refd = conv.double_backward(prob, rowptr, col, vec, x, th, g, r32(W.normal(x.shape, 62)),
                                r32(W.normal(vec.shape, 63)), r32(W.normal(th.shape, 64) * 0.05))
    assert rel(dbl["d_g"].cpu().numpy(), refd["d_g"]) < TOL[gemm]


def test_validate_mode_rejects_bad_graphs(T):
    """validate=1: the graph is checked on the device before any stream kernel
    reads it; a sender index out of range, a broken rowptr or a zero-length edge
    vector returns TPCONV_ERR_GRAPH_INVALID, a good graph runs normally."""
    import torch
    rowptr, col, vec = W.graph_for("tiny", 0)
    irr = "8x0e+8x1o"
    plan = T.Plan(irr, 2, irr, 4, radial="gaussian", radial_params=(0.5, 5.0), validate=True)
    prob = conv.Problem(irr, 2, irr, 4, "gaussian", (0.5, 5.0))
    N = len(rowptr) - 1
    x = W.normal((N, prob.dim_in), 71)
    th = W.theta([(4 * p.c_in * p.c_out, 0.2) for p in prob.paths], 72)
    xd, thd = dev(x, torch.float32), dev(th, torch.float32)
    good = T.Graph(dev(rowptr, torch.int32), dev(col, torch.int32), dev(vec, torch.float32))
    out = T.forward(plan, good, xd, thd)
    torch.cuda.synchronize()
    ref = conv.forward(prob, rowptr, col, vec.astype(np.float32).astype(np.float64), x.astype(np.float32),
                       th.astype(np.float32))
    assert rel(out.cpu().numpy(), ref) < TOL_FP32
    bad_col = col.copy()
    bad_col[5] = N + 3
    bad_rp = rowptr.copy()
    bad_rp[7], bad_rp[8] = bad_rp[8], bad_rp[7] - 1
    bad_vec = vec.copy()
    bad_vec[11] = 0.0
    for rp_, col_, vec_ in ((rowptr, bad_col, vec), (bad_rp, col, vec), (rowptr, col, bad_vec)):
        G = T.Graph(dev(rp_, torch.int32), dev(col_, torch.int32), dev(vec_, torch.float32))
        with pytest.raises(T.TPConvError) as e:
            T.forward(plan, G, xd, thd)
        assert e.value.status == 6  # TPCONV_ERR_GRAPH_INVALID
