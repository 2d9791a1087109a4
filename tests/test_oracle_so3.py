"""Pins for the oracle's spherical harmonics, generators and CG tensors.

Every check compares against something the mathematics fixes independently of
the oracle's construction: the textbook real-SH table, quadrature
orthonormality, the addition theorem, parity, finite differences, the so(3)
algebra, Gaunt integrals and the 1o x 1o couplings (dot and cross product).
"""

import math

import numpy as np
import pytest

from oracle import so3


def _pts(n, seed=0):
    g = np.random.default_rng(seed)
    v = g.normal(size=(n, 3))
    return v * g.uniform(0.5, 3.0, size=(n, 1))


def test_sh_textbook_table_l_le_3():
    # Standard table of real spherical harmonics (orthonormal, no Condon-Shortley
    # sign), times sqrt(4 pi) for component normalisation; m = -l..l.
    v = _pts(50, 1)
    n = v / np.linalg.norm(v, axis=1, keepdims=True)
    x, y, z = n.T
    s4p = math.sqrt(4 * math.pi)
    table = {
        0: [0.5 * math.sqrt(1 / math.pi) + 0 * x],
        1: [math.sqrt(3 / (4 * math.pi)) * y, math.sqrt(3 / (4 * math.pi)) * z,
            math.sqrt(3 / (4 * math.pi)) * x],
        2: [0.5 * math.sqrt(15 / math.pi) * x * y, 0.5 * math.sqrt(15 / math.pi) * y * z,
            0.25 * math.sqrt(5 / math.pi) * (3 * z * z - 1), 0.5 * math.sqrt(15 / math.pi) * x * z,
            0.25 * math.sqrt(15 / math.pi) * (x * x - y * y)],
        3: [0.25 * math.sqrt(35 / (2 * math.pi)) * y * (3 * x * x - y * y),
            0.5 * math.sqrt(105 / math.pi) * x * y * z,
            0.25 * math.sqrt(21 / (2 * math.pi)) * y * (5 * z * z - 1),
            0.25 * math.sqrt(7 / math.pi) * z * (5 * z * z - 3),
            0.25 * math.sqrt(21 / (2 * math.pi)) * x * (5 * z * z - 1),
            0.25 * math.sqrt(105 / math.pi) * z * (x * x - y * y),
            0.25 * math.sqrt(35 / (2 * math.pi)) * x * (x * x - 3 * y * y)],
    }
    for l, rows in table.items():
        want = s4p * np.stack(rows, axis=-1)
        np.testing.assert_allclose(so3.real_sh(l, v), want, atol=1e-13)


@pytest.mark.parametrize("l", range(7))
def test_sh_addition_theorem_and_parity(l):
    v = _pts(40, l)
    Y = so3.real_sh(l, v)
    np.testing.assert_allclose((Y ** 2).sum(-1), 2 * l + 1, rtol=1e-12)
    np.testing.assert_allclose(so3.real_sh(l, -v), (-1) ** l * Y, atol=1e-12)
    np.testing.assert_allclose(so3.real_sh(l, 3.7 * v), Y, atol=1e-12)


def test_sh_orthonormal_by_quadrature():
    pts, w = so3.sphere_quadrature(16, 32)
    Y = so3.sh_all(6, pts)
    G = np.einsum('q,qa,qb->ab', w, Y, Y)
    np.testing.assert_allclose(G, 4 * np.pi * np.eye(Y.shape[1]), atol=1e-11)


@pytest.mark.parametrize("l", range(5))
def test_sh_gradient_and_hessian_fd(l):
    v = _pts(6, 10 + l)
    h = 1e-5
    G = so3.real_sh_grad(l, v)
    H = so3.real_sh_hess(l, v)
    for i in range(3):
        dv = np.zeros(3)
        dv[i] = h
        fd = (so3.real_sh(l, v + dv) - so3.real_sh(l, v - dv)) / (2 * h)
        np.testing.assert_allclose(G[..., i], fd, atol=1e-8)
        fdg = (so3.real_sh_grad(l, v + dv) - so3.real_sh_grad(l, v - dv)) / (2 * h)
        np.testing.assert_allclose(H[..., :, i], fdg, atol=1e-7)
    np.testing.assert_allclose(H, np.swapaxes(H, -1, -2), atol=1e-12)


@pytest.mark.parametrize("l", range(1, 7))
def test_generators_so3_algebra(l):
    J = so3.generators(l)
    for a in range(3):
        np.testing.assert_allclose(J[a], -J[a].T, atol=1e-12)
    # [J_x, J_y] = J_z and cyclic (matching [K_x, K_y] = K_z for K_a v = e_a x v)
    for a, b, c in [(0, 1, 2), (1, 2, 0), (2, 0, 1)]:
        np.testing.assert_allclose(J[a] @ J[b] - J[b] @ J[a], J[c], atol=1e-11)
    cas = sum(J[a] @ J[a] for a in range(3))
    np.testing.assert_allclose(cas, -l * (l + 1) * np.eye(2 * l + 1), atol=1e-10)


@pytest.mark.parametrize("l", range(5))
def test_wigner_two_constructions(l):
    g = np.random.default_rng(3 + l)
    axis, ang = g.normal(size=3), g.uniform(0, 2 * np.pi)
    Q = so3.rotation_from_axis_angle(axis, ang)
    np.testing.assert_allclose(Q @ Q.T, np.eye(3), atol=1e-13)
    D1 = so3.wigner_D_lstsq(l, Q)
    D2 = so3.wigner_D_expm(l, axis, ang)
    np.testing.assert_allclose(D1, D2, atol=1e-11)
    np.testing.assert_allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-11)
    np.testing.assert_allclose(so3.wigner_D_lstsq(l, -np.eye(3)), (-1) ** l * np.eye(2 * l + 1),
                               atol=1e-12)


def _triples(lmax):
    return [(a, b, c) for a in range(lmax + 1) for b in range(lmax + 1) for c in range(lmax + 1)
            if abs(a - b) <= c <= a + b]


@pytest.mark.parametrize("t", _triples(3))
def test_cg_orthogonality_and_equivariance(t):
    l1, l2, l3 = t
    C = so3.real_cg(*t)
    np.testing.assert_allclose(np.einsum('abk,abq->kq', C, C), np.eye(2 * l3 + 1), atol=1e-12)
    g = np.random.default_rng(sum(t))
    Q = so3.rotation_from_axis_angle(g.normal(size=3), g.uniform(0, 6))
    D1, D2, D3 = (so3.wigner_D_lstsq(l, Q) for l in t)
    x, y = g.normal(size=2 * l1 + 1), g.normal(size=2 * l2 + 1)
    lhs = np.einsum('abk,a,b->k', C, D1 @ x, D2 @ y)
    rhs = D3 @ np.einsum('abk,a,b->k', C, x, y)
    np.testing.assert_allclose(lhs, rhs, atol=1e-11)


@pytest.mark.parametrize("l1,l2", [(a, b) for a in range(4) for b in range(4)])
def test_cg_completeness(l1, l2):
    n = (2 * l1 + 1) * (2 * l2 + 1)
    S = np.zeros((n, n))
    for l3 in range(abs(l1 - l2), l1 + l2 + 1):
        C = so3.real_cg(l1, l2, l3).reshape(n, -1)
        S += C @ C.T
    np.testing.assert_allclose(S, np.eye(n), atol=1e-12)


def test_cg_closed_forms():
    for l in range(4):
        np.testing.assert_allclose(so3.real_cg(0, l, l)[0], np.eye(2 * l + 1), atol=1e-13)
        np.testing.assert_allclose(so3.real_cg(l, 0, l)[:, 0, :], np.eye(2 * l + 1), atol=1e-13)
    # 1o x 1o -> 0e is the dot product
    np.testing.assert_allclose(so3.real_cg(1, 1, 0)[:, :, 0], np.eye(3) / math.sqrt(3), atol=1e-13)
    # 1o x 1o -> 1e is the antisymmetric cross product, components in (y, z, x) order
    eps = np.zeros((3, 3, 3))
    for (a, b, c), s in {(0, 1, 2): 1, (1, 2, 0): 1, (2, 0, 1): 1,
                         (1, 0, 2): -1, (2, 1, 0): -1, (0, 2, 1): -1}.items():
        eps[a, b, c] = s
    np.testing.assert_allclose(so3.real_cg(1, 1, 1), eps / math.sqrt(2), atol=1e-13)
    # nonzero counts
    nnz = {t: int((np.abs(so3.real_cg(*t)) > 1e-10).sum())
           for t in [(1, 1, 2), (2, 2, 2), (3, 3, 3), (3, 3, 6)]}
    assert nnz == {(1, 1, 2): 11, (2, 2, 2): 25, (3, 3, 3): 42, (3, 3, 6): 79}


@pytest.mark.parametrize("t", [t for t in _triples(3) if sum(t) % 2 == 0])
def test_cg_proportional_to_gaunt(t):
    """For even l1+l2+l3 the real CG is a multiple of the Gaunt integral
    int Y_l1m1 Y_l2m2 Y_l3m3 dOmega, computed here by exact quadrature."""
    pts, w = so3.sphere_quadrature(12, 24)
    G = np.einsum('q,qa,qb,qc->abc', w, so3.real_sh(t[0], pts), so3.real_sh(t[1], pts),
                  so3.real_sh(t[2], pts))
    C = so3.real_cg(*t)
    kappa = (G * C).sum() / (C * C).sum()
    assert abs(kappa) > 1e-6
    np.testing.assert_allclose(G, kappa * C, atol=1e-11)
    # and the SH product identity: sum C Y_l1 Y_l2 is proportional to Y_l3 everywhere
    v = _pts(20, 7)
    lhs = np.einsum('abc,qa,qb->qc', C, so3.real_sh(t[0], v), so3.real_sh(t[1], v))
    ratio = kappa / (4 * np.pi)   # coefficient of Y_l3 in Y_l1 Y_l2 is G / (4 pi)
    np.testing.assert_allclose(lhs, ratio * so3.real_sh(t[2], v), atol=1e-11)


def test_cg_symmetry_under_swap():
    # C^{l l L}[a, b, c] = (-1)^(2l - L) C^{l l L}[b, a, c] (symmetric for even L)
    for l in range(4):
        for L in range(0, 2 * l + 1):
            C = so3.real_cg(l, l, L)
            np.testing.assert_allclose(C, (-1) ** (2 * l - L) * np.swapaxes(C, 0, 1), atol=1e-12)
