"""Real spherical harmonics, so(3) generators and real Clebsch-Gordan tensors.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Conventions (readings; the pages print no formulas):

* Real basis, m = -l..l.  m < 0 are sine-type, m > 0 cosine-type; no
  Condon-Shortley sign in the real functions, so Y_1 is proportional to
  (y, z, x) in that order.
* "Component" normalisation: Y_l(n) = sqrt(4 pi) * (orthonormal real SH), so
  sum_m Y_lm(n)^2 = 2l+1 and Y_0 = 1.
* Y_l(v) for a non-unit vector v means Y_l(v / |v|).

Real SH are built from the Cartesian closed form of real solid harmonics
(Legendre part Pi_l^m(z) times the azimuthal polynomials A_m / B_m), kept as
exact polynomial coefficient tables so that gradients and Hessians are exact
polynomial derivatives.

The Clebsch-Gordan tensor C[m1, m2, m3] of a triple (l1, l2, l3) is *not*
taken from the Racah formula here: it is the one-dimensional null space of
the infinitesimal intertwiner equations

    C(J1 x, y) + C(x, J2 y) = J3 C(x, y)    for the three generators J_a,

where the real-basis generators J_a of degree l are read off the spherical
harmonics themselves (d/dt Y_l(exp(t K_a) n) = J_a Y_l(n)).  It is then
normalised so that sum_{m1 m2} C[m1,m2,m3] C[m1,m2,m3'] = delta_{m3 m3'} and
its sign fixed so that the first entry (lexicographic m1, m2, m3) whose
magnitude exceeds 1e-9 is positive.  This is the coupling of "The Price of
Freedom" (Approach: Clebsch-Gordan tensor product, selection rules).
"""

from __future__ import annotations

import functools
import math

import numpy as np

# --------------------------------------------------------------------------
# exact polynomials in (x, y, z):  dict {(a, b, c): coefficient}
# --------------------------------------------------------------------------


def _padd(p, q, s=1.0):
    out = dict(p)
    for k, v in q.items():
        out[k] = out.get(k, 0.0) + s * v
    return {k: v for k, v in out.items() if v != 0.0}


def _pmul(p, q):
    out = {}
    for (a1, b1, c1), v1 in p.items():
        for (a2, b2, c2), v2 in q.items():
            k = (a1 + a2, b1 + b2, c1 + c2)
            out[k] = out.get(k, 0.0) + v1 * v2
    return {k: v for k, v in out.items() if v != 0.0}


def _pscale(p, s):
    return {k: v * s for k, v in p.items() if v * s != 0.0}


def _pdiff(p, i):
    out = {}
    for k, v in p.items():
        if k[i] == 0:
            continue
        nk = list(k)
        nk[i] -= 1
        nk = tuple(nk)
        out[nk] = out.get(nk, 0.0) + v * k[i]
    return out


def _peval(p, v):
    """Evaluate polynomial p at points v[..., 3]."""
    x, y, z = v[..., 0], v[..., 1], v[..., 2]
    out = np.zeros(v.shape[:-1], dtype=np.float64)
    for (a, b, c), coef in p.items():
        out = out + coef * (x ** a) * (y ** b) * (z ** c)
    return out


def _r2_pow(k):
    """(x^2 + y^2 + z^2)^k expanded."""
    out = {(0, 0, 0): 1.0}
    r2 = {(2, 0, 0): 1.0, (0, 2, 0): 1.0, (0, 0, 2): 1.0}
    for _ in range(k):
        out = _pmul(out, r2)
    return out


_COS_QUARTER = (1.0, 0.0, -1.0, 0.0)  # cos(q*pi/2), q mod 4
_SIN_QUARTER = (0.0, 1.0, 0.0, -1.0)  # sin(q*pi/2), q mod 4


@functools.lru_cache(maxsize=None)
def sh_polys(l: int):
    """Homogeneous degree-l polynomials P_lm with Y_lm(n) = P_lm(n) on |n| = 1.

    Component normalisation (times sqrt(4 pi) relative to orthonormal).
    Returned as a tuple of 2l+1 coefficient dicts, m = -l..l.
    """
    polys = []
    for m in range(-l, l + 1):
        am = abs(m)
        # Legendre part Pi_l^{|m|}(z, r)
        pi_lm = {}
        for k in range((l - am) // 2 + 1):
            c = ((-1) ** k) * 2.0 ** (-l) * math.comb(l, k) * math.comb(2 * l - 2 * k, l) \
                * math.factorial(l - 2 * k) / math.factorial(l - 2 * k - am)
            term = _pmul(_r2_pow(k), {(0, 0, l - 2 * k - am): c})
            pi_lm = _padd(pi_lm, term)
        pi_lm = _pscale(pi_lm, math.sqrt(math.factorial(l - am) / math.factorial(l + am)))
        # azimuthal part
        az = {}
        for p in range(am + 1):
            q = (am - p) % 4
            trig = _COS_QUARTER[q] if m >= 0 else _SIN_QUARTER[q]
            if trig != 0.0:
                az = _padd(az, {(p, am - p, 0): math.comb(am, p) * trig})
        if m == 0:
            norm = math.sqrt((2 * l + 1) / (4 * math.pi))
        else:
            norm = math.sqrt((2 * l + 1) / (2 * math.pi))
        poly = _pscale(_pmul(pi_lm, az), norm * math.sqrt(4 * math.pi))
        polys.append(poly)
    return tuple(polys)


def real_sh(l: int, v: np.ndarray) -> np.ndarray:
    """Y_l(v / |v|), shape (..., 2l+1)."""
    v = np.asarray(v, dtype=np.float64)
    n = v / np.linalg.norm(v, axis=-1, keepdims=True)
    return np.stack([_peval(p, n) for p in sh_polys(l)], axis=-1)


def real_sh_grad(l: int, v: np.ndarray) -> np.ndarray:
    """d Y_lm / d v_i, shape (..., 2l+1, 3).

    With Y(v) = P(v) / |v|^l:  grad Y = grad P / r^l - l P v / r^(l+2).
    """
    v = np.asarray(v, dtype=np.float64)
    r = np.linalg.norm(v, axis=-1)
    out = []
    for p in sh_polys(l):
        P = _peval(p, v)
        g = np.stack([_peval(_pdiff(p, i), v) for i in range(3)], axis=-1)
        out.append(g / r[..., None] ** l - l * (P / r ** (l + 2))[..., None] * v)
    return np.stack(out, axis=-2)


def real_sh_hess(l: int, v: np.ndarray) -> np.ndarray:
    """d^2 Y_lm / d v_i d v_j, shape (..., 2l+1, 3, 3).

    For f = P r^-l:  f_ij = P_ij r^-l - l r^-(l+2) (P_i v_j + P_j v_i)
                            - l r^-(l+2) P delta_ij + l (l+2) r^-(l+4) P v_i v_j.
    """
    v = np.asarray(v, dtype=np.float64)
    r = np.linalg.norm(v, axis=-1)
    eye = np.eye(3)
    out = []
    for p in sh_polys(l):
        P = _peval(p, v)
        dP = [_pdiff(p, i) for i in range(3)]
        g = np.stack([_peval(d, v) for d in dP], axis=-1)
        H = np.stack([np.stack([_peval(_pdiff(dP[i], j), v) for j in range(3)], axis=-1)
                      for i in range(3)], axis=-2)
        rl = r[..., None, None]
        t = H / rl ** l
        t = t - l / rl ** (l + 2) * (g[..., :, None] * v[..., None, :] + v[..., :, None] * g[..., None, :])
        t = t - l * (P / r ** (l + 2))[..., None, None] * eye
        t = t + l * (l + 2) * (P / r ** (l + 4))[..., None, None] * (v[..., :, None] * v[..., None, :])
        out.append(t)
    return np.stack(out, axis=-3)


def sh_all(lmax: int, v):
    """Concatenated Y_0..Y_lmax, shape (..., (lmax+1)^2)."""
    return np.concatenate([real_sh(l, v) for l in range(lmax + 1)], axis=-1)


def sh_all_grad(lmax: int, v):
    return np.concatenate([real_sh_grad(l, v) for l in range(lmax + 1)], axis=-2)


def sh_all_hess(lmax: int, v):
    return np.concatenate([real_sh_hess(l, v) for l in range(lmax + 1)], axis=-3)


# --------------------------------------------------------------------------
# sphere quadrature (Gauss-Legendre in cos(theta) x uniform in phi)
# --------------------------------------------------------------------------


def sphere_quadrature(n_theta: int, n_phi: int):
    """Points n[q, 3] and weights w[q] with sum w = 4 pi; exact for
    polynomials of degree < min(2 n_theta, n_phi) restricted to the sphere."""
    ct, wt = np.polynomial.legendre.leggauss(n_theta)
    phi = 2 * np.pi * np.arange(n_phi) / n_phi
    st = np.sqrt(1 - ct ** 2)
    pts = np.stack([st[:, None] * np.cos(phi)[None, :],
                    st[:, None] * np.sin(phi)[None, :],
                    np.broadcast_to(ct[:, None], (n_theta, n_phi))], axis=-1).reshape(-1, 3)
    w = np.broadcast_to(wt[:, None] * (2 * np.pi / n_phi), (n_theta, n_phi)).reshape(-1)
    return pts, w.copy()


# --------------------------------------------------------------------------
# generators and Clebsch-Gordan null space
# --------------------------------------------------------------------------

_K = np.array([  # K_a v = e_a x v
    [[0, 0, 0], [0, 0, -1], [0, 1, 0]],
    [[0, 0, 1], [0, 0, 0], [-1, 0, 0]],
    [[0, -1, 0], [1, 0, 0], [0, 0, 0]],
], dtype=np.float64)


@functools.lru_cache(maxsize=None)
def generators(l: int) -> np.ndarray:
    """Real-basis generators J[a] (a = x, y, z) of degree l: grad Y_l(n) . (K_a n) = J_a Y_l(n).

    Projected with exact quadrature using  int Y_lm Y_lm' dOmega = 4 pi delta.
    """
    pts, w = sphere_quadrature(2 * l + 4, 4 * l + 8)
    Y = real_sh(l, pts)                      # (q, 2l+1)
    G = real_sh_grad(l, pts)                 # (q, 2l+1, 3)
    J = np.zeros((3, 2 * l + 1, 2 * l + 1))
    for a in range(3):
        kn = pts @ _K[a].T                   # (q, 3)  = K_a n
        dY = np.einsum('qmi,qi->qm', G, kn)  # (q, 2l+1)
        J[a] = np.einsum('q,qm,qk->mk', w, dY, Y) / (4 * np.pi)
    return J


def triangle_ok(l1: int, l2: int, l3: int) -> bool:
    return abs(l1 - l2) <= l3 <= l1 + l2


@functools.lru_cache(maxsize=None)
def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """Real Clebsch-Gordan tensor C[m1, m2, m3] (fp64), null-space construction."""
    if not triangle_ok(l1, l2, l3):
        raise ValueError(f"triangle rule violated for ({l1},{l2},{l3})")
    n1, n2, n3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    J1, J2, J3 = generators(l1), generators(l2), generators(l3)
    I1, I2, I3 = np.eye(n1), np.eye(n2), np.eye(n3)
    rows = []
    for a in range(3):
        rows.append(np.kron(np.kron(J1[a].T, I2), I3)
                    + np.kron(np.kron(I1, J2[a].T), I3)
                    - np.kron(np.kron(I1, I2), J3[a]))
    L = np.concatenate(rows, axis=0)
    _, s, vt = np.linalg.svd(L)
    # the intertwiner space of an allowed triple is one-dimensional
    if s[-1] > 1e-9 or (len(s) > 1 and s[-2] < 1e-6):
        raise RuntimeError(f"unexpected null space for ({l1},{l2},{l3}): {s[-3:]}")
    c = vt[-1].reshape(n1, n2, n3)
    c = c * math.sqrt(n3) / np.linalg.norm(c)
    flat = c.reshape(-1)
    first = np.flatnonzero(np.abs(flat) > 1e-9)[0]
    if flat[first] < 0:
        c = -c
    c[np.abs(c) < 1e-13] = 0.0
    return c


# --------------------------------------------------------------------------
# Wigner D matrices (two constructions; used by the equivariance tests)
# --------------------------------------------------------------------------


def wigner_D_lstsq(l: int, Q: np.ndarray, rng=None) -> np.ndarray:
    """D_l(Q) fitted from Y_l(Q n) = D_l(Q) Y_l(n) on random points.

    Q may be improper; then D carries the (-1)^l of Y_l(-n)."""
    rng = np.random.default_rng(12345) if rng is None else rng
    n = rng.normal(size=(8 * (2 * l + 1) + 16, 3))
    A = real_sh(l, n)            # (q, 2l+1)
    B = real_sh(l, n @ Q.T)      # (q, 2l+1)  rows: Y(Q n_q)
    # B = A D^T
    Dt, *_ = np.linalg.lstsq(A, B, rcond=None)
    return Dt.T


def _expm_antisym(M: np.ndarray) -> np.ndarray:
    """exp(M) by scaling and squaring of a Taylor series (small matrices)."""
    nrm = np.linalg.norm(M, 1)
    k = max(0, int(math.ceil(math.log2(max(nrm, 1e-300)))) + 4)
    A = M / (2 ** k)
    out = np.eye(M.shape[0])
    term = np.eye(M.shape[0])
    for i in range(1, 30):
        term = term @ A / i
        out = out + term
    for _ in range(k):
        out = out @ out
    return out


def rotation_from_axis_angle(axis, angle):
    axis = np.asarray(axis, dtype=np.float64)
    axis = axis / np.linalg.norm(axis)
    K = np.einsum('a,aij->ij', axis, _K)
    return _expm_antisym(angle * K)


def wigner_D_expm(l: int, axis, angle) -> np.ndarray:
    """D_l(exp(angle * axis . K)) = exp(angle * axis . J_l)  (proper rotations)."""
    axis = np.asarray(axis, dtype=np.float64)
    axis = axis / np.linalg.norm(axis)
    J = np.einsum('a,aij->ij', axis, generators(l))
    return _expm_antisym(angle * J)
