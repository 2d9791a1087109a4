"""The torch module over the C ABI: first- and second-order autograd (forces
and their gradients) against the fp64 oracle."""

import numpy as np
import pytest

import workloads as W
from oracle import conv

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-5


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    d = np.abs(b).max()
    return np.abs(a - b).max() / (d if d > 0 else 1.0)


@pytest.mark.parametrize("name", ["tiny", "radius_small"])
def test_module_first_and_second_order_autograd(name):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import equivariant_gnn_tensor_receiver_b200 as T
    if name == "tiny":
        irr, lsh, R, rad, rp = "8x0e+8x1o", 2, 4, "gaussian", (0.5, 5.0)
        rowptr, col, vec = W.graph_for("tiny", 3)
    else:
        irr, lsh, R, rad, rp = "16x0e+16x1o+16x2e", 3, 8, "bessel", (5.0,)
        rowptr, col, vec = W.radius_graph(300, 14.0, 5.0, 9)
    torch.manual_seed(0)
    m = T.TPConv(irr, lsh, irr, R, radial=rad, radial_params=rp)
    prob = conv.Problem(irr, lsh, irr, R, rad, rp)
    N = len(rowptr) - 1
    d = lambda a, t=torch.float32: torch.as_tensor(np.ascontiguousarray(a), dtype=t, device="cuda")
    v = d(vec).requires_grad_(True)
    G = T.Graph(d(rowptr, torch.int32), d(col, torch.int32), v)
    x = d(W.normal((N, prob.dim_in), 31)).requires_grad_(True)
    f32 = lambda a: a.astype(np.float32).astype(np.float64)  # what the device sees
    w = f32(W.normal((N, prob.dim_out), 32))
    cx, cv = f32(W.normal((N, prob.dim_in), 33)), f32(W.normal(vec.shape, 34))
    out = m(x, G)
    energy = (out * d(w)).sum()
    dx, dth, dvec = torch.autograd.grad(energy, [x, m.theta, v], create_graph=True)
    loss = (dx * d(cx)).sum() + (dvec * d(cv)).sum()
    gx, gth, gv = torch.autograd.grad(loss, [x, m.theta, v])
    r32 = lambda a: a.detach().double().cpu().numpy()
    x64, th64, v64 = r32(x), r32(m.theta), r32(v)
    ref_out = conv.forward(prob, rowptr, col, v64, x64, th64)
    assert rel(r32(out), ref_out) < TOL_FP32
    rb = conv.backward(prob, rowptr, col, v64, x64, th64, w)
    for got, k in ((dx, "dx"), (dth, "dtheta"), (dvec, "dvec")):
        assert rel(r32(got), rb[k]) < TOL_FP32, k
    rd = conv.double_backward(prob, rowptr, col, v64, x64, th64, w, cx, cv, None)
    for got, k in ((gx, "d_x"), (gth, "d_theta"), (gv, "d_vec")):
        assert rel(r32(got), rd[k]) < TOL_FP32, k
