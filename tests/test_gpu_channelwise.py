"""GPU parity of the channel-wise operator family against the oracle, through
the C ABI: forward, backward and double backward on small graphs (every output
element), the mace-sized layer on sampled receivers, edges and senders, and
the node-side state in chunks (workspace cap).

Tolerance: the fp32 bar of the other parity tests (max-norm relative error
1e-5).  The edge streams are those of the full family; the node-level sums
are plain fp32 FMAs over R x paths terms.
"""

import numpy as np
import pytest

import workloads as W
from oracle import conv

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-5


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


CASES = {
    # name: (irreps_in, lsh, irreps_out, R, radial, params, graph)
    "tiny": ("8x0e+8x1o", 2, "8x0e+8x1o", 4, "gaussian", (0.5, 5.0), lambda: W.graph_for("tiny", 0)),
    "mixed_l3": ("4x0e+4x1o+4x1e+4x2e+4x3o", 3, "4x0e+4x0o+4x1o+4x2e+4x3o", 3, "bessel", (5.0,),
                 lambda: W.random_graph(40, 400, 5, r_min=0.6, r_max=4.8)),
    # channel counts that are not a multiple of 4 take the per-path edge streams
    "odd_channels": ("3x0e+3x1o", 2, "3x0e+3x1o", 5, "bessel", (5.0,),
                     lambda: W.random_graph(25, 180, 8, r_min=0.6, r_max=4.8)),
    "radius_small": ("16x0e+16x1o+16x2e", 3, "16x0e+16x1o+16x2e", 8, "bessel", (5.0,),
                     lambda: W.radius_graph(300, 14.0, 5.0, 7)),
}


def make(T, case, seed, cap=0, graph=None):
    import torch
    irr_in, lsh, irr_out, R, rad, rp, gf = CASES[case] if isinstance(case, str) else case
    rowptr, col, vec = graph if graph is not None else gf()
    plan = T.Plan(irr_in, lsh, irr_out, R, radial=rad, radial_params=rp, workspace_cap=cap, family="channelwise")
    prob = conv.Problem(irr_in, lsh, irr_out, R, rad, rp, family="channelwise")
    N = len(rowptr) - 1
    r32 = lambda a: a.astype(np.float32).astype(np.float64)
    x = r32(W.normal((N, prob.dim_in), seed + 1))
    th = r32(W.theta([(R * p.c_in, 1.0 / np.sqrt(R)) for p in prob.paths], seed + 2))
    g = r32(W.normal((N, prob.dim_out), seed + 3))
    G = T.Graph(dev(rowptr, torch.int32), dev(col, torch.int32), dev(vec, torch.float32))
    return plan, prob, G, (rowptr, col, r32(vec), x, th, g)


@pytest.mark.parametrize("cap", [0, 1])
@pytest.mark.parametrize("case", list(CASES))
def test_forward_backward_parity(T, case, cap):
    import torch
    plan, prob, G, (rowptr, col, vec, x, th, g) = make(T, case, 11)
    if cap:  # node-side state in chunks of about a fifth of the nodes
        N = len(rowptr) - 1
        afl = sum(prob.R * p.c_in * (2 * p.l3 + 1) for p in prob.paths)   # receiver state floats per node
        bfl = sum(prob.R * p.c_out * (2 * p.l1 + 1) for p in prob.paths)  # sender state floats per node
        plan = T.Plan(*CASES[case][:4], radial=CASES[case][4], radial_params=CASES[case][5],
                      workspace_cap=max(1, N // 5) * max(afl, bfl) * 4, family="channelwise")
    xd, thd, gd = dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32)
    out = T.forward(plan, G, xd, thd)
    bw = T.backward(plan, G, xd, thd, gd, want=("dx", "dtheta", "dvec", "dY", "db"))
    torch.cuda.synchronize()
    ref = conv.forward(prob, rowptr, col, vec, x, th)
    assert rel(out.cpu().numpy(), ref) < TOL_FP32
    rb = conv.backward(prob, rowptr, col, vec, x, th, g)
    for k in ("dx", "dtheta", "dvec", "dY", "db"):
        assert rel(bw[k].cpu().numpy(), rb[k]) < TOL_FP32, (k, rel(bw[k].cpu().numpy(), rb[k]))


@pytest.mark.parametrize("case,which", [("tiny", "xvt"), ("mixed_l3", "xvt"), ("odd_channels", "xvt"),
                                        ("radius_small", "xv"), ("mixed_l3", "t")])
def test_double_backward_parity(T, case, which):
    import torch
    plan, prob, G, (rowptr, col, vec, x, th, g) = make(T, case, 51)
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


def test_mace_full_size_sampled(T):
    """The mace-sized layer (4096 atoms, ~214k edges) with channel-wise weights:
    forward on sampled receivers, d_vec on their edges, dx on sampled senders,
    each computed by the oracle from exactly the edges involved; dTheta via the
    identity <dTheta, D> = directional derivative, which holds at any size."""
    import torch
    c = W.CONFIGS["mace"]
    case = (c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"], tuple(c["radial_params"]), None)
    plan, prob, G, (rowptr, col, vec, x, th, g) = make(T, case, 41, graph=W.graph_for("mace", 0))
    xd, thd, gd = dev(x, torch.float32), dev(th, torch.float32), dev(g, torch.float32)
    out = T.forward(plan, G, xd, thd).cpu().numpy()
    bw = {k: v.cpu().numpy() for k, v in
          T.backward(plan, G, xd, thd, gd, want=("dx", "dtheta", "dvec")).items()}
    torch.cuda.synchronize()
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    rs = np.random.default_rng(0).choice(N, 24, replace=False)
    em = np.isin(recv, rs)
    loc = {r: i for i, r in enumerate(rs)}
    lr = np.array([loc[r] for r in recv[em]])
    Y, b, JY, Jb = conv.geometry(prob, vec[em], order=1)
    ref = conv.forward_core(prob, len(rs), col[em].astype(np.int64), lr, x, Y, b, th)
    assert rel(out[rs], ref) < TOL_FP32
    _, _, dY, db = conv.backward_core(prob, len(rs), col[em].astype(np.int64), lr, x, Y, b, th, g[rs])
    dvec = np.einsum('em,emi->ei', dY, JY) + np.einsum('ek,eki->ei', db, Jb)
    assert rel(bw["dvec"][em], dvec) < TOL_FP32
    ss = np.random.default_rng(1).choice(N, 16, replace=False)
    sm = np.isin(col, ss)
    Y2, b2 = conv.geometry(prob, vec[sm])
    dx, _, _, _ = conv.backward_core(prob, N, col[sm].astype(np.int64), recv[sm], x, Y2, b2, th, g)
    assert rel(bw["dx"][ss], dx[ss]) < TOL_FP32
    # <dTheta, D> = <g, forward(x, D)>: the forward is linear in Theta
    D = W.normal(th.shape, 77).astype(np.float32)
    lhs = float(np.dot(bw["dtheta"].astype(np.float64), D.astype(np.float64)))
    fD = T.forward(plan, G, xd, dev(D, torch.float32)).double().cpu().numpy()
    terms = g * fD
    assert abs(lhs - terms.sum()) <= TOL_FP32 * (np.abs(terms).sum() + np.abs(bw["dtheta"] * D).sum())


def test_torch_module_channelwise(T):
    """TPConv(family="channelwise"): forces (d out / d vec) and their Theta gradient against the oracle."""
    import torch
    irr_in, lsh, irr_out, R, rad, rp, gf = CASES["tiny"]
    rowptr, col, vec = gf()
    m = T.TPConv(irr_in, lsh, irr_out, R, radial=rad, radial_params=rp, family="channelwise")
    prob = conv.Problem(irr_in, lsh, irr_out, R, rad, rp, family="channelwise")
    assert m.theta.numel() == prob.theta_numel
    N = len(rowptr) - 1
    x = torch.tensor(W.normal((N, prob.dim_in), 3), dtype=torch.float32, device="cuda")
    v = torch.tensor(vec, dtype=torch.float32, device="cuda", requires_grad=True)
    G = T.Graph(dev(rowptr, torch.int32), dev(col, torch.int32), v)
    gw = torch.tensor(W.normal((N, prob.dim_out), 4), dtype=torch.float32, device="cuda")
    out = m(x, G)
    (fv,) = torch.autograd.grad((out * gw).sum(), v, create_graph=True)
    cv = torch.tensor(W.normal(vec.shape, 5), dtype=torch.float32, device="cuda")
    (fv * cv).sum().backward()
    th = m.theta.detach().double().cpu().numpy()
    xs, gs, vs = (a.double().cpu().numpy() for a in (x, gw, v.detach()))
    rb = conv.backward(prob, rowptr, col, vs, xs, th, gs)
    assert rel(fv.detach().cpu().numpy(), rb["dvec"]) < TOL_FP32
    rd = conv.double_backward(prob, rowptr, col, vs, xs, th, gs, None, cv.double().cpu().numpy(), None)
    assert rel(m.theta.grad.cpu().numpy(), rd["d_theta"]) < TOL_FP32
