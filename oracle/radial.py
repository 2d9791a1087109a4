"""Radial bases b_k(r) and their first two derivatives (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name a "radial projection" (Sobek, abstract) but print no basis.
Readings, one per workload family:

* Gaussian:  b_k(r) = exp(-((r - mu_k) / D)^2),  mu_k = r_min + k D,
             D = (r_max - r_min) / (R - 1),  k = 0..R-1  (D = r_max - r_min if R = 1).
* Bessel with cosine cutoff:
             b_k(r) = sqrt(2 / r_c) sin(k pi r / r_c) / r * (cos(pi r / r_c) + 1) / 2,
             k = 1..R, and 0 for r >= r_c.

Each function returns (b, db/dr, d2b/dr2), each of shape (..., R).
"""

from __future__ import annotations

import numpy as np


def gaussian(r, R: int, r_min: float, r_max: float):
    r = np.asarray(r, dtype=np.float64)[..., None]
    D = (r_max - r_min) / (R - 1) if R > 1 else (r_max - r_min)
    mu = r_min + D * np.arange(R)
    t = (r - mu) / D
    b = np.exp(-t * t)
    d1 = -2.0 * t / D * b
    d2 = (4.0 * t * t - 2.0) / (D * D) * b
    return b, d1, d2


def bessel_cos(r, R: int, r_cut: float):
    r = np.asarray(r, dtype=np.float64)[..., None]
    k = np.arange(1, R + 1)
    a = k * np.pi / r_cut
    pre = np.sqrt(2.0 / r_cut)
    s, c = np.sin(a * r), np.cos(a * r)
    f = pre * s / r                                   # sin(a r) / r part
    f1 = pre * (a * c / r - s / r ** 2)
    f2 = pre * (-a * a * s / r - 2.0 * a * c / r ** 2 + 2.0 * s / r ** 3)
    w = np.pi / r_cut
    fc = 0.5 * (np.cos(w * r) + 1.0)
    fc1 = -0.5 * w * np.sin(w * r)
    fc2 = -0.5 * w * w * np.cos(w * r)
    inside = (r < r_cut).astype(np.float64)
    b = f * fc * inside
    d1 = (f1 * fc + f * fc1) * inside
    d2 = (f2 * fc + 2.0 * f1 * fc1 + f * fc2) * inside
    return b, d1, d2


def evaluate(kind: str, r, R: int, params: tuple):
    if kind == "gaussian":
        return gaussian(r, R, *params)
    if kind == "bessel":
        return bessel_cos(r, R, *params)
    raise ValueError(kind)


def vector_derivs(kind: str, v, R: int, params: tuple):
    """b(|v|) with gradient (..., R, 3) and Hessian (..., R, 3, 3) in v."""
    v = np.asarray(v, dtype=np.float64)
    r = np.linalg.norm(v, axis=-1)
    b, d1, d2 = evaluate(kind, r, R, params)
    u = v / r[..., None]
    grad = d1[..., :, None] * u[..., None, :]
    uu = u[..., :, None] * u[..., None, :]
    proj = (np.eye(3) - uu) / r[..., None, None]
    hess = d2[..., :, None, None] * uu[..., None, :, :] + d1[..., :, None, None] * proj[..., None, :, :]
    return b, grad, hess
