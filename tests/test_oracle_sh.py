"""Pins of the oracle's real spherical harmonics and of the Wigner-D tool.

Convention (LunaTP, arXiv 2610.18393, Table 1 edge irreps 1x0e+1x1o+...;
the pages fix no normalisation, so the plain component normalisation is
taken): sum_m Y_lm^2 = 2l+1, order m=-l..l, no Condon-Shortley phase,
Y_1 = sqrt3 (y, z, x).
"""
import numpy as np
import pytest
import scipy.special as sps

import oracle as O
from tests._so3 import random_rotation, wigner_d

L = 6


def _unit(rng, n):
    v = rng.standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def test_degree_one_is_sqrt3_yzx():
    rng = np.random.default_rng(0)
    r = rng.standard_normal((20, 3)) * 3.0
    Y = O.sph_harm(1, r)
    u = r / np.linalg.norm(r, axis=1, keepdims=True)
    assert np.allclose(Y[:, 0], 1.0, atol=1e-15)
    assert np.allclose(Y[:, 1:4], np.sqrt(3) * u[:, [1, 2, 0]], atol=1e-14)


def test_z_axis_values():
    Y = O.sph_harm(L, [[0, 0, 2.5]])[0]
    for l in range(L + 1):
        blk = Y[l * l:(l + 1) ** 2]
        assert blk[l] == pytest.approx(np.sqrt(2 * l + 1), abs=1e-13)
        assert np.allclose(np.delete(blk, l), 0.0, atol=1e-13)


def test_component_normalisation():
    rng = np.random.default_rng(1)
    Y = O.sph_harm(L, _unit(rng, 50))
    for l in range(L + 1):
        s = (Y[:, l * l:(l + 1) ** 2] ** 2).sum(1)
        assert np.allclose(s, 2 * l + 1, atol=1e-12)


def test_addition_theorem():
    # sum_m Y_lm(a) Y_lm(b) = (2l+1) P_l(a.b) with component normalisation
    rng = np.random.default_rng(2)
    a, b = _unit(rng, 40), _unit(rng, 40)
    Ya, Yb = O.sph_harm(L, a), O.sph_harm(L, b)
    c = (a * b).sum(1)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) ** 2)
        lhs = (Ya[:, sl] * Yb[:, sl]).sum(1)
        rhs = (2 * l + 1) * sps.eval_legendre(l, c)
        assert np.allclose(lhs, rhs, atol=1e-12)


def test_parity():
    rng = np.random.default_rng(3)
    r = _unit(rng, 30)
    Yp, Ym = O.sph_harm(L, r), O.sph_harm(L, -r)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) ** 2)
        assert np.allclose(Ym[:, sl], (-1) ** l * Yp[:, sl], atol=1e-12)


def test_quadrature_orthogonality():
    # int Y_lm Y_l'm' dOmega = 4 pi delta, Gauss-Legendre in cos(theta) x
    # trapezoid in phi, exact for these degrees
    nth, nph = 16, 32
    ct, wt = np.polynomial.legendre.leggauss(nth)
    ph = np.arange(nph) * 2 * np.pi / nph
    st = np.sqrt(1 - ct ** 2)
    P = np.stack([np.outer(st, np.cos(ph)).ravel(), np.outer(st, np.sin(ph)).ravel(),
                  np.repeat(ct, nph)], axis=1)
    w = np.repeat(wt, nph) * (2 * np.pi / nph)
    Y = O.sph_harm(L, P)
    G = (Y * w[:, None]).T @ Y
    assert np.allclose(G, 4 * np.pi * np.eye(G.shape[0]), atol=1e-11)


def test_matches_scipy_complex_harmonics():
    # library routine: scipy's complex Y_l^m (orthonormal, with Condon-Shortley
    # phase) mapped to the real basis:
    #   m>0: sqrt2 (-1)^m Re Y_l^m ; m<0: sqrt2 (-1)^m Im Y_l^|m| ; times sqrt(4 pi)
    rng = np.random.default_rng(4)
    r = _unit(rng, 25)
    th = np.arccos(np.clip(r[:, 2], -1, 1))
    ph = np.arctan2(r[:, 1], r[:, 0])
    Y = O.sph_harm(L, r)
    for l in range(L + 1):
        for m in range(-l, l + 1):
            c = sps.sph_harm_y(l, abs(m), th, ph) * np.sqrt(4 * np.pi)
            if m == 0:
                ref = c.real
            elif m > 0:
                ref = np.sqrt(2) * (-1) ** m * c.real
            else:
                ref = np.sqrt(2) * (-1) ** m * c.imag
            assert np.allclose(Y[:, l * l + l + m], ref, atol=1e-12), (l, m)


def test_zero_vector():
    Y = O.sph_harm(3, [[0.0, 0.0, 0.0]])[0]
    assert Y[0] == 1.0 and np.all(Y[1:] == 0.0)


def test_wigner_d_is_a_representation():
    rng = np.random.default_rng(5)
    R1, R2 = random_rotation(rng), random_rotation(rng)
    assert np.allclose(R1 @ R1.T, np.eye(3)) and np.linalg.det(R1) == pytest.approx(1.0)
    for l in range(L + 1):
        D1, D2, D12 = wigner_d(l, R1), wigner_d(l, R2), wigner_d(l, R1 @ R2)
        assert np.allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-11)
        assert np.linalg.det(D1) == pytest.approx(1.0, abs=1e-10)
        assert np.allclose(D12, D1 @ D2, atol=1e-11)
        if l == 1:  # in the (y, z, x) ordering D^1 is R permuted
            perm = [1, 2, 0]
            assert np.allclose(D1, R1[np.ix_(perm, perm)], atol=1e-12)
