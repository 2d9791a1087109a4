"""Pins for the oracle's radial bases: closed values, cutoff, derivatives."""

import math

import numpy as np

from oracle import radial


def test_gaussian_values():
    r = np.array([0.5, 2.0, 5.0])
    b, _, _ = radial.gaussian(r, 4, 0.5, 5.0)
    # centres 0.5, 2.0, 3.5, 5.0 with width 1.5
    np.testing.assert_allclose(np.diag(b[:, [0, 1, 3]]), 1.0)
    np.testing.assert_allclose(b[1, 2], math.exp(-1.0))
    np.testing.assert_allclose(b[0, 3], math.exp(-9.0))


def test_bessel_values_and_cutoff():
    r = np.array([1.0, 2.5, 5.0, 6.0])
    b, d1, _ = radial.bessel_cos(r, 3, 5.0)
    want = math.sqrt(2 / 5) * math.sin(math.pi * 1.0 / 5) / 1.0 * 0.5 * (math.cos(math.pi / 5) + 1)
    np.testing.assert_allclose(b[0, 0], want)
    # k = 2 vanishes at r = r_c / 2; everything vanishes at and beyond r_c
    np.testing.assert_allclose(b[1, 1], 0.0, atol=1e-15)
    assert np.all(b[2:] == 0) and np.all(d1[2:] == 0)


def test_derivatives_fd():
    r = np.linspace(0.6, 4.8, 17)
    h = 1e-6
    for f in (lambda t: radial.gaussian(t, 5, 0.5, 5.0), lambda t: radial.bessel_cos(t, 8, 5.0)):
        b, d1, d2 = f(r)
        np.testing.assert_allclose(d1, (f(r + h)[0] - f(r - h)[0]) / (2 * h), rtol=1e-6, atol=1e-8)
        np.testing.assert_allclose(d2, (f(r + h)[1] - f(r - h)[1]) / (2 * h), rtol=1e-6, atol=1e-7)


def test_vector_derivatives_fd():
    g = np.random.default_rng(0)
    v = g.normal(size=(5, 3))
    v *= g.uniform(0.8, 4.0, size=(5, 1)) / np.linalg.norm(v, axis=1, keepdims=True)
    h = 1e-6
    for kind, params in (("bessel", (5.0,)), ("gaussian", (0.5, 5.0))):
        b, G, H = radial.vector_derivs(kind, v, 6, params)
        for i in range(3):
            dv = np.zeros(3)
            dv[i] = h
            bp, Gp, _ = radial.vector_derivs(kind, v + dv, 6, params)
            bm, Gm, _ = radial.vector_derivs(kind, v - dv, 6, params)
            np.testing.assert_allclose(G[..., i], (bp - bm) / (2 * h), atol=1e-8)
            np.testing.assert_allclose(H[..., :, i], (Gp - Gm) / (2 * h), atol=1e-7)
