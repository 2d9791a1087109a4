"""Pins for the oracle's convolution (forward, backward, double backward).

Checks against facts fixed by the mathematics, not by the oracle's own code:
selection-rule path counts, O(3) equivariance with Wigner-D matrices fitted
from the spherical harmonics, closed forms of special cases (SpMM, dot
product, cross product), a dense brute-force bilinear form, finite
differences, torch fp64 autograd of an independently written forward,
linearity, relabelling and chunk additivity.
"""

import math

import numpy as np
import pytest

import workloads as W
from oracle import conv, irreps, radial, so3


def _problem(name, **kw):
    c = dict(W.CONFIGS[name])
    c.update(kw)
    return conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                        tuple(c["radial_params"]))


def _small(seed=0, N=7, E=19, irr_in="2x0e+2x1o+1x2e", lsh=2, irr_out="1x0e+2x1o+2x2e", R=3,
           rad="bessel", rp=(5.0,)):
    prob = conv.Problem(irr_in, lsh, irr_out, R, rad, rp)
    rowptr, col, vec = W.random_graph(N, E, seed, r_min=0.6, r_max=4.4)
    x = W.normal((N, prob.dim_in), seed + 1)
    th = W.normal(prob.theta_numel, seed + 2)
    return prob, rowptr, col, vec, x, th


def test_path_counts_per_config():
    counts = {k: len(_problem(k).paths) for k in ("tiny", "mace", "sweep", "wide")}
    assert counts == {"tiny": 5, "mace": 13, "sweep": 11, "wide": 23}
    ps = _problem("tiny").paths
    assert [(p.l1, p.l2, p.l3) for p in ps] == [(0, 0, 0), (1, 1, 0), (0, 1, 1), (1, 0, 1), (1, 2, 1)]
    mace = {(p.l1, p.l2, p.l3) for p in _problem("mace").paths}
    assert mace == {(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0), (1, 2, 1), (0, 2, 2), (1, 1, 2),
                    (1, 3, 2), (2, 0, 2), (2, 1, 1), (2, 2, 0), (2, 2, 2), (2, 3, 1)}
    assert _problem("mace").theta_numel == 425984


def _block_D(blocks, Q, improper):
    mats = []
    for b in blocks:
        D = so3.wigner_D_lstsq(b.l, Q)   # includes (-1)^l when Q is improper
        if improper:
            # a block of parity p picks up p under inversion; Y_l already gave (-1)^l
            D = D * (b.p * (-1) ** b.l)
        mats += [D] * b.mul
    n = sum(m.shape[0] for m in mats)
    out = np.zeros((n, n))
    o = 0
    for m in mats:
        k = m.shape[0]
        out[o:o + k, o:o + k] = m
        o += k
    return out


@pytest.mark.parametrize("improper", [False, True])
@pytest.mark.parametrize("case", ["tiny", "mixed"])
def test_equivariance_O3(case, improper):
    if case == "tiny":
        prob = _problem("tiny")
        rowptr, col, vec = W.random_graph(20, 60, 4)
        x = W.normal((20, prob.dim_in), 5)
    else:
        prob = conv.Problem("2x0e+1x1o+2x1e+1x2e+1x3o", 3, "1x0o+2x1e+1x1o+2x2e+1x3e+1x3o", 2,
                            "bessel", (5.0,))
        rowptr, col, vec = W.random_graph(15, 50, 6, r_min=0.6, r_max=4.0)
        x = W.normal((15, prob.dim_in), 7)
    assert len(prob.paths) > 0
    th = W.normal(prob.theta_numel, 8)
    g = np.random.default_rng(9)
    Q = so3.rotation_from_axis_angle(g.normal(size=3), g.uniform(0, 6))
    if improper:
        Q = -Q
    Din = _block_D(irreps.parse(prob.irreps_in), Q, improper)
    Dout = _block_D(irreps.parse(prob.irreps_out), Q, improper)
    out = conv.forward(prob, rowptr, col, vec, x, th)
    out_rot = conv.forward(prob, rowptr, col, vec @ Q.T, x @ Din.T, th)
    err = np.abs(out_rot - out @ Dout.T).max() / np.abs(out).max()
    assert err < 1e-10


def test_special_case_spmm():
    """0e only, SH l=0, R=1, Theta=I: out = A_b x with A_b[r, s] = sum_e b(|v_e|)."""
    prob = conv.Problem("5x0e", 0, "5x0e", 1, "bessel", (5.0,))
    rowptr, col, vec = W.random_graph(30, 200, 11, r_min=0.6, r_max=4.5)
    x = W.normal((30, 5), 12)
    th = np.eye(5).reshape(-1)
    recv = np.repeat(np.arange(30), np.diff(rowptr))
    r = np.linalg.norm(vec, axis=1)
    b = math.sqrt(2 / 5.0) * np.sin(math.pi * r / 5.0) / r * 0.5 * (np.cos(math.pi * r / 5.0) + 1)
    A = np.zeros((30, 30))
    np.add.at(A, (recv, col), b)
    np.testing.assert_allclose(conv.forward(prob, rowptr, col, vec, x, th), A @ x, rtol=1e-12,
                               atol=1e-12)


def _closed(kind):
    rowptr, col, vec = W.random_graph(25, 90, 13, r_min=0.6, r_max=4.5)
    recv = np.repeat(np.arange(25), np.diff(rowptr))
    n = vec / np.linalg.norm(vec, axis=1, keepdims=True)
    n_yzx = n[:, [1, 2, 0]]
    r = np.linalg.norm(vec, axis=1)
    b = np.exp(-((r - 0.5) / 4.5) ** 2)  # Gaussian basis, R = 1, on [0.5, 5]
    return rowptr, col, vec, recv, n_yzx, b


def test_special_case_dot_product():
    """1o -> 0e through l2 = 1 is b * (x_s . v_hat), features in (y, z, x) order."""
    rowptr, col, vec, recv, n, b = _closed("dot")
    prob = conv.Problem("1x1o", 1, "1x0e", 1, "gaussian", (0.5, 5.0))
    x = W.normal((25, 3), 14)
    want = np.zeros((25, 1))
    np.add.at(want[:, 0], recv, b * (x[col] * n).sum(1))
    np.testing.assert_allclose(conv.forward(prob, rowptr, col, vec, x, np.ones(1)), want, atol=1e-12)


def test_special_case_scalar_times_direction():
    """0e -> 1o through l2 = 1 is sqrt(3) b x_s v_hat."""
    rowptr, col, vec, recv, n, b = _closed("vec")
    prob = conv.Problem("1x0e", 1, "1x1o", 1, "gaussian", (0.5, 5.0))
    x = W.normal((25, 1), 15)
    want = np.zeros((25, 3))
    np.add.at(want, recv, math.sqrt(3) * b[:, None] * x[col] * n)
    np.testing.assert_allclose(conv.forward(prob, rowptr, col, vec, x, np.ones(1)), want, atol=1e-12)


def test_special_case_cross_product():
    """1o -> 1e through l2 = 1 is sqrt(3/2) b (x_s x v_hat) -- the antisymmetric
    coupling that separates chiral shapes (The Price of Freedom, Key results)."""
    rowptr, col, vec, recv, n, b = _closed("cross")
    prob = conv.Problem("1x1o", 1, "1x1e", 1, "gaussian", (0.5, 5.0))
    x = W.normal((25, 3), 16)
    xs = x[col][:, [2, 0, 1]]            # back to (x, y, z)
    nn = n[:, [2, 0, 1]]
    cr = np.cross(xs, nn)[:, [1, 2, 0]]  # to (y, z, x)
    want = np.zeros((25, 3))
    np.add.at(want, recv, math.sqrt(1.5) * b[:, None] * cr)
    np.testing.assert_allclose(conv.forward(prob, rowptr, col, vec, x, np.ones(1)), want, atol=1e-12)


def test_brute_force_dense_bilinear():
    prob, rowptr, col, vec, x, th = _small(seed=20)
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    Y = so3.sh_all(prob.l_sh_max, vec)
    b, _, _ = radial.evaluate(prob.radial, np.linalg.norm(vec, axis=1), prob.R, prob.radial_params)
    want = np.zeros((N, prob.dim_out))
    for e in range(len(col)):
        M = np.zeros((prob.dim_in, prob.n_sh, prob.dim_out))
        for p in prob.paths:
            C = so3.real_cg(p.l1, p.l2, p.l3)
            Wp = np.tensordot(b[e], prob.theta_block(th, p), axes=1)
            n1, n2, n3 = 2 * p.l1 + 1, 2 * p.l2 + 1, 2 * p.l3 + 1
            for u in range(p.c_in):
                for w in range(p.c_out):
                    for a in range(n1):
                        for c in range(n3):
                            M[p.in_off + u * n1 + a, p.l2 ** 2:p.l2 ** 2 + n2,
                              p.out_off + w * n3 + c] += C[a, :, c] * Wp[u, w]
        want[recv[e]] += np.einsum('i,j,ijo->o', x[col[e]], Y[e], M)
    np.testing.assert_allclose(conv.forward(prob, rowptr, col, vec, x, th), want, rtol=1e-12,
                               atol=1e-12)


def test_linearity_and_relabelling():
    prob, rowptr, col, vec, x, th = _small(seed=30)
    N = len(rowptr) - 1
    x2 = W.normal(x.shape, 31)
    th2 = W.normal(th.shape, 32)
    f = lambda xx, tt: conv.forward(prob, rowptr, col, vec, xx, tt)
    np.testing.assert_allclose(f(2 * x - 3 * x2, th), 2 * f(x, th) - 3 * f(x2, th), atol=1e-11)
    np.testing.assert_allclose(f(x, th + th2), f(x, th) + f(x, th2), atol=1e-11)
    # relabel nodes with a permutation pi: node i -> pi[i]
    pi = np.random.default_rng(33).permutation(N)
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    send2, recv2 = pi[col], pi[recv]
    order = np.argsort(recv2, kind="stable")
    rp2 = np.zeros(N + 1, dtype=np.int64)
    np.cumsum(np.bincount(recv2, minlength=N), out=rp2[1:])
    x_p = np.empty_like(x)
    x_p[pi] = x
    out_p = conv.forward(prob, rp2, send2[order], vec[order], x_p, th)
    np.testing.assert_allclose(out_p[pi], f(x, th), atol=1e-11)


def test_chunk_additivity_of_dtheta():
    """Splitting receivers into two ranges and summing dTheta reproduces dTheta."""
    prob, rowptr, col, vec, x, th = _small(seed=40, N=12, E=40)
    N = len(rowptr) - 1
    g = W.normal((N, prob.dim_out), 41)
    full = conv.backward(prob, rowptr, col, vec, x, th, g)["dtheta"]
    cut = 5
    parts = []
    for lo, hi in ((0, cut), (cut, N)):
        gm = np.zeros_like(g)
        gm[lo:hi] = g[lo:hi]
        parts.append(conv.backward(prob, rowptr, col, vec, x, th, gm)["dtheta"])
    np.testing.assert_allclose(parts[0] + parts[1], full, atol=1e-11)


def _fd(f, z, dz, h=1e-6):
    return (f(z + h * dz) - f(z - h * dz)) / (2 * h)


@pytest.mark.parametrize("rad", [("bessel", (5.0,)), ("gaussian", (0.5, 5.0))])
def test_backward_matches_finite_differences(rad):
    prob, rowptr, col, vec, x, th = _small(seed=50, rad=rad[0], rp=rad[1])
    N = len(rowptr) - 1
    g = W.normal((N, prob.dim_out), 51)
    bw = conv.backward(prob, rowptr, col, vec, x, th, g)
    L = lambda xx, vv, tt: (g * conv.forward(prob, rowptr, col, vv, xx, tt)).sum()
    rng = np.random.default_rng(52)
    for _ in range(3):
        dxd, dvd, dtd = rng.normal(size=x.shape), rng.normal(size=vec.shape), rng.normal(size=th.shape)
        np.testing.assert_allclose(_fd(lambda z: L(z, vec, th), x, dxd), (bw["dx"] * dxd).sum(),
                                   rtol=1e-7)
        np.testing.assert_allclose(_fd(lambda z: L(x, z, th), vec, dvd), (bw["dvec"] * dvd).sum(),
                                   rtol=1e-7)
        np.testing.assert_allclose(_fd(lambda z: L(x, vec, z), th, dtd), (bw["dtheta"] * dtd).sum(),
                                   rtol=1e-7)


@pytest.mark.parametrize("which", ["all", "no_theta"])
def test_double_backward_matches_finite_differences(which):
    prob, rowptr, col, vec, x, th = _small(seed=60)
    N = len(rowptr) - 1
    rng = np.random.default_rng(61)
    g = rng.normal(size=(N, prob.dim_out))
    ggx, ggv = rng.normal(size=x.shape), rng.normal(size=vec.shape)
    ggt = rng.normal(size=th.shape) if which == "all" else None

    def psi(gg, xx, vv, tt):
        bw = conv.backward(prob, rowptr, col, vv, xx, tt, gg)
        s = (ggx * bw["dx"]).sum() + (ggv * bw["dvec"]).sum()
        if ggt is not None:
            s += (ggt * bw["dtheta"]).sum()
        return s

    db = conv.double_backward(prob, rowptr, col, vec, x, th, g, ggx, ggv, ggt)
    for _ in range(2):
        d = [rng.normal(size=a.shape) for a in (g, x, vec, th)]
        np.testing.assert_allclose(_fd(lambda z: psi(z, x, vec, th), g, d[0]), (db["d_g"] * d[0]).sum(),
                                   rtol=1e-6)
        np.testing.assert_allclose(_fd(lambda z: psi(g, z, vec, th), x, d[1]), (db["d_x"] * d[1]).sum(),
                                   rtol=1e-6)
        np.testing.assert_allclose(_fd(lambda z: psi(g, x, z, th), vec, d[2]),
                                   (db["d_vec"] * d[2]).sum(), rtol=1e-6)
        np.testing.assert_allclose(_fd(lambda z: psi(g, x, vec, z), th, d[3]),
                                   (db["d_theta"] * d[3]).sum(), rtol=1e-6, atol=1e-9)


def test_torch_autograd_cross_check():
    """fp64 torch autograd of a separately written dense forward (SH from the
    textbook table, so only l <= 3) must give the oracle's backward and double
    backward."""
    torch = pytest.importorskip("torch")
    prob, rowptr, col, vec, x, th = _small(seed=70, irr_in="2x0e+1x1o+1x2e", lsh=3,
                                           irr_out="1x0e+1x1o+2x2e", R=2)
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    rng = np.random.default_rng(71)
    g = rng.normal(size=(N, prob.dim_out))
    ggx, ggv, ggt = rng.normal(size=x.shape), rng.normal(size=vec.shape), rng.normal(size=th.shape)
    T = lambda a: torch.tensor(a, dtype=torch.float64)

    def sh_table(v):
        r = torch.linalg.norm(v, dim=1, keepdim=True)
        xx, yy, zz = (v / r).unbind(1)
        s = math.sqrt
        rows = [torch.ones_like(xx),
                s(3) * yy, s(3) * zz, s(3) * xx,
                s(15) * xx * yy, s(15) * yy * zz, s(5) / 2 * (3 * zz * zz - 1), s(15) * xx * zz,
                s(15) / 2 * (xx * xx - yy * yy),
                s(70) / 4 * yy * (3 * xx * xx - yy * yy), s(105) * xx * yy * zz,
                s(42) / 4 * yy * (5 * zz * zz - 1), s(7) / 2 * zz * (5 * zz * zz - 3),
                s(42) / 4 * xx * (5 * zz * zz - 1), s(105) / 2 * zz * (xx * xx - yy * yy),
                s(70) / 4 * xx * (xx * xx - 3 * yy * yy)]
        return torch.stack(rows, 1)

    def bessel(v):
        r = torch.linalg.norm(v, dim=1, keepdim=True)
        k = torch.arange(1, prob.R + 1, dtype=torch.float64)
        return math.sqrt(2 / 5.0) * torch.sin(k * math.pi * r / 5.0) / r * 0.5 * (
            torch.cos(math.pi * r / 5.0) + 1)

    def fwd(xt, vt, tt, gt):
        Y, b = sh_table(vt), bessel(vt)
        out = torch.zeros(N, prob.dim_out, dtype=torch.float64)
        for p in prob.paths:
            C = T(so3.real_cg(p.l1, p.l2, p.l3))
            n1, n3 = 2 * p.l1 + 1, 2 * p.l3 + 1
            xs = xt[col, p.in_off:p.in_off + p.c_in * n1].reshape(-1, p.c_in, n1)
            Wt = torch.einsum('ek,kuw->euw', b, tt[p.theta_off:p.theta_off + prob.R * p.c_in * p.c_out]
                              .reshape(prob.R, p.c_in, p.c_out))
            msg = torch.einsum('ijk,eui,ej,euw->ewk', C, xs, Y[:, p.l2 ** 2:(p.l2 + 1) ** 2], Wt)
            out = out.index_add(0, torch.as_tensor(recv),
                                torch.nn.functional.pad(msg.reshape(len(col), -1),
                                                        (p.out_off, prob.dim_out - p.out_off - p.c_out * n3)))
        return (out * gt).sum()

    xt, vt, tt, gt = (T(a).requires_grad_() for a in (x, vec, th, g))
    L = fwd(xt, vt, tt, gt)
    dx, dv, dt = torch.autograd.grad(L, (xt, vt, tt), create_graph=True)
    bw = conv.backward(prob, rowptr, col, vec, x, th, g)
    np.testing.assert_allclose(dx.detach().numpy(), bw["dx"], atol=1e-11)
    np.testing.assert_allclose(dv.detach().numpy(), bw["dvec"], atol=1e-11)
    np.testing.assert_allclose(dt.detach().numpy(), bw["dtheta"], atol=1e-11)
    psi = (dx * T(ggx)).sum() + (dv * T(ggv)).sum() + (dt * T(ggt)).sum()
    d2 = torch.autograd.grad(psi, (gt, xt, vt, tt))
    db = conv.double_backward(prob, rowptr, col, vec, x, th, g, ggx, ggv, ggt)
    for got, key in zip(d2, ("d_g", "d_x", "d_vec", "d_theta")):
        np.testing.assert_allclose(got.numpy(), db[key], atol=1e-10, err_msg=key)
