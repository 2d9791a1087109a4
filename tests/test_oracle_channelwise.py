"""Pins for the oracle's channel-wise operator family.

The channel-wise product keeps every channel on its own: W_e[p] is the
diagonal matrix diag(sum_k b_ek Theta[p][k, :]).  It is therefore the full
(fully connected) product evaluated at the block-diagonal Theta_full[p][k] =
diag(Theta[p][k]), and the full product is pinned on its own
(``test_oracle_conv.py``: equivariance, closed forms, finite differences,
torch autograd).  These tests hold the channel-wise code to that special case
at every differentiation order, with the gradient in Theta being the diagonal
of the full gradient.  They also check one edge by brute force (explicit loops
over channels and m), the Theta layout, and the rejection of paths whose
input and output multiplicities differ.
"""

import numpy as np
import pytest

import workloads as W
from oracle import conv, so3


def _case(seed=3, N=6, E=17, irr_in="3x0e+3x1o+3x2e", lsh=2, irr_out="3x0e+3x1o+3x2e", R=3):
    cw = conv.Problem(irr_in, lsh, irr_out, R, "bessel", (5.0,), family="channelwise")
    full = conv.Problem(irr_in, lsh, irr_out, R, "bessel", (5.0,))
    rowptr, col, vec = W.random_graph(N, E, seed, r_min=0.6, r_max=4.4)
    x = W.normal((N, cw.dim_in), seed + 1)
    th = W.normal(cw.theta_numel, seed + 2)
    return cw, full, rowptr, col, vec, x, th


def _diag_full(cw, full, th):
    """Theta_full[p][k] = diag(Theta[p][k, :])."""
    out = np.zeros(full.theta_numel)
    for pc, pf in zip(cw.paths, full.paths):
        blk = cw.theta_block(th, pc)                      # (R, C)
        d = np.zeros((cw.R, pc.c_in, pc.c_out))
        for k in range(cw.R):
            d[k] = np.diag(blk[k])
        out[pf.theta_off:pf.theta_off + d.size] = d.reshape(-1)
    return out


def _diag_of(cw, full, dfull):
    """The diagonal of a full-layout Theta gradient, in the channel-wise layout."""
    out = np.zeros(cw.theta_numel)
    for pc, pf in zip(cw.paths, full.paths):
        blk = dfull[pf.theta_off:pf.theta_off + cw.R * pc.c_in * pc.c_out].reshape(cw.R, pc.c_in, pc.c_out)
        out[pc.theta_off:pc.theta_off + cw.R * pc.c_in] = np.stack([np.diag(blk[k]) for k in range(cw.R)]).reshape(-1)
    return out


def test_theta_layout_and_sizes():
    c = W.CONFIGS["mace"]
    cw = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], family="channelwise")
    assert len(cw.paths) == 13
    assert cw.theta_numel == 13 * 8 * 64                   # R x C per path
    assert [p.theta_off for p in cw.paths] == [512 * i for i in range(13)]


def test_unequal_multiplicities_rejected():
    with pytest.raises(ValueError):
        conv.Problem("4x0e+2x1o", 1, "3x0e+2x1o", 2, family="channelwise")
    with pytest.raises(ValueError):
        conv.Problem("4x0e", 1, "4x0e", 2, family="depthwise")


def test_forward_is_full_product_at_diagonal_theta():
    cw, full, rowptr, col, vec, x, th = _case()
    a = conv.forward(cw, rowptr, col, vec, x, th)
    b = conv.forward(full, rowptr, col, vec, x, _diag_full(cw, full, th))
    assert np.abs(a).max() > 0.1
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_forward_one_edge_by_brute_force():
    """One edge, explicit loops: out[r, i3, u, m3] = sum_p sum_k b_k Theta[p][k,u] sum C x Y."""
    cw, _, _, _, _, x, th = _case()
    N = x.shape[0]
    rowptr = np.array([0, 0, 1] + [1] * (N - 2), dtype=np.int64)   # one edge into node 1
    col = np.array([4])
    vec = np.array([[0.7, -1.1, 2.0]])
    out = conv.forward(cw, rowptr, col, vec, x, th)
    Y, b = conv.geometry(cw, vec)
    ref = np.zeros(cw.dim_out)
    for p in cw.paths:
        C = so3.real_cg(p.l1, p.l2, p.l3)
        n1, n2, n3 = 2 * p.l1 + 1, 2 * p.l2 + 1, 2 * p.l3 + 1
        T = th[p.theta_off:p.theta_off + cw.R * p.c_in].reshape(cw.R, p.c_in)
        for u in range(p.c_in):
            w = sum(b[0, k] * T[k, u] for k in range(cw.R))
            for m3 in range(n3):
                acc = 0.0
                for m1 in range(n1):
                    for m2 in range(n2):
                        acc += C[m1, m2, m3] * x[4, p.in_off + u * n1 + m1] * Y[0, p.l2 ** 2 + m2]
                ref[p.out_off + u * n3 + m3] += w * acc
    np.testing.assert_allclose(out[1], ref, rtol=1e-12, atol=1e-12)
    assert np.abs(np.delete(out, 1, axis=0)).max() == 0


def test_backward_is_full_adjoint_at_diagonal_theta():
    cw, full, rowptr, col, vec, x, th = _case(seed=5)
    g = W.normal((x.shape[0], cw.dim_out), 9)
    a = conv.backward(cw, rowptr, col, vec, x, th, g)
    b = conv.backward(full, rowptr, col, vec, x, _diag_full(cw, full, th), g)
    for k in ("dx", "dvec", "dY", "db"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(a["dtheta"], _diag_of(cw, full, b["dtheta"]), rtol=1e-12, atol=1e-12)


def test_dtheta_by_finite_differences():
    cw, _, rowptr, col, vec, x, th = _case(seed=8)
    g = W.normal((x.shape[0], cw.dim_out), 10)
    dth = conv.backward(cw, rowptr, col, vec, x, th, g)["dtheta"]
    h = 1e-6
    for i in (0, 5, cw.theta_numel // 2, cw.theta_numel - 1):
        e = np.zeros_like(th)
        e[i] = h
        fd = (np.sum(g * conv.forward(cw, rowptr, col, vec, x, th + e))
              - np.sum(g * conv.forward(cw, rowptr, col, vec, x, th - e))) / (2 * h)
        assert abs(fd - dth[i]) <= 1e-7 * max(1.0, abs(fd))


def test_double_backward_is_full_at_diagonal_theta():
    cw, full, rowptr, col, vec, x, th = _case(seed=11)
    N, E = x.shape[0], len(col)
    g = W.normal((N, cw.dim_out), 12)
    gx = W.normal((N, cw.dim_in), 13)
    gv = W.normal((E, 3), 14)
    gt = W.normal(cw.theta_numel, 15)
    a = conv.double_backward(cw, rowptr, col, vec, x, th, g, gx, gv, gt)
    b = conv.double_backward(full, rowptr, col, vec, x, _diag_full(cw, full, th), g, gx, gv,
                             _diag_full(cw, full, gt))
    for k in ("d_g", "d_x", "d_vec"):
        np.testing.assert_allclose(a[k], b[k], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(a["d_theta"], _diag_of(cw, full, b["d_theta"]), rtol=1e-11, atol=1e-11)
