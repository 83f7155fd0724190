"""Pins of the oracle's Clebsch-Gordan tables.

The complex coefficients come from Racah's closed form; they are pinned to
textbook special values, to sympy's exact CG (a library routine) and to
orthonormality.  The real coefficients, in the basis of the oracle's real
spherical harmonics, are pinned by the intertwiner identity with Wigner-D
matrices fitted from those harmonics (so any mismatch between the two bases
fails), by orthonormality and by the three identity couplings.
"""
import itertools

import numpy as np
import pytest

import oracle as O
from tests._so3 import random_rotation, wigner_d


@pytest.mark.parametrize("args,val", [
    ((1, 0, 1, 0, 0, 0), -1 / np.sqrt(3)),
    ((1, 1, 1, -1, 2, 0), 1 / np.sqrt(6)),
    ((1, 0, 1, 0, 2, 0), np.sqrt(2 / 3)),
    ((1, 1, 1, 0, 1, 1), 1 / np.sqrt(2)),
    ((2, 2, 3, 3, 5, 5), 1.0),           # stretched state
    ((3, 1, 0, 0, 3, 1), 1.0),           # coupling to l=0
])
def test_textbook_values(args, val):
    assert O.cg_complex(*args) == pytest.approx(val, abs=1e-14)


def test_singlet_closed_form():
    # <l m l -m | 0 0> = (-1)^(l-m) / sqrt(2l+1)
    for l in range(7):
        for m in range(-l, l + 1):
            assert O.cg_complex(l, m, l, -m, 0, 0) == pytest.approx(
                (-1) ** (l - m) / np.sqrt(2 * l + 1), abs=1e-14)


def test_matches_sympy_exact():
    from sympy.physics.quantum.cg import CG
    for j1, j2 in itertools.product(range(4), range(4)):
        for J in range(abs(j1 - j2), j1 + j2 + 1):
            for m1 in range(-j1, j1 + 1):
                for m2 in range(-j2, j2 + 1):
                    M = m1 + m2
                    if abs(M) > J:
                        continue
                    ref = float(CG(j1, m1, j2, m2, J, M).doit())
                    assert O.cg_complex(j1, m1, j2, m2, J, M) == pytest.approx(ref, abs=1e-13)


def test_sympy_spot_checks_high_l():
    from sympy.physics.quantum.cg import CG
    for (j1, m1, j2, m2, J) in [(6, 2, 6, -1, 7), (5, -3, 6, 4, 6), (6, 6, 6, -6, 0), (4, 1, 6, -2, 3)]:
        ref = float(CG(j1, m1, j2, m2, J, m1 + m2).doit())
        assert O.cg_complex(j1, m1, j2, m2, J, m1 + m2) == pytest.approx(ref, abs=1e-13)


def test_complex_orthonormality():
    for j1, j2 in [(1, 1), (2, 3), (4, 4), (6, 5)]:
        for J, Jp in itertools.product(range(abs(j1 - j2), j1 + j2 + 1), repeat=2):
            for M in range(-min(J, Jp), min(J, Jp) + 1):
                s = sum(O.cg_complex(j1, m1, j2, M - m1, J, M) * O.cg_complex(j1, m1, j2, M - m1, Jp, M)
                        for m1 in range(-j1, j1 + 1) if abs(M - m1) <= j2)
                assert s == pytest.approx(1.0 if J == Jp else 0.0, abs=1e-12)


def _triples(lmax):
    for l1, l2 in itertools.product(range(lmax + 1), repeat=2):
        for l3 in range(abs(l1 - l2), min(l1 + l2, lmax) + 1):
            yield l1, l2, l3


def test_real_orthonormality_and_sign():
    for l1, l2, l3 in _triples(6):
        C = O.real_cg(l1, l2, l3)
        G = np.einsum("abi,abj->ij", C, C)
        assert np.allclose(G, np.eye(2 * l3 + 1), atol=1e-12), (l1, l2, l3)
        flat = C.ravel()
        first = flat[np.abs(flat) > 1e-12][0]
        assert first > 0


def test_real_identity_couplings():
    for l in range(7):
        n = 2 * l + 1
        assert np.allclose(O.real_cg(0, l, l)[0], np.eye(n), atol=1e-13)
        assert np.allclose(O.real_cg(l, 0, l)[:, 0, :], np.eye(n), atol=1e-13)
        assert np.allclose(O.real_cg(l, l, 0)[:, :, 0], np.eye(n) / np.sqrt(n), atol=1e-13)


def test_triangle_rule_rejected():
    with pytest.raises(ValueError):
        O.real_cg(1, 1, 3)


def test_real_intertwiner_identity():
    # (D^l1 (x) D^l2) C = C D^l3 : the coupled vector rotates with D^l3
    rng = np.random.default_rng(11)
    for _ in range(2):
        R = random_rotation(rng)
        D = [wigner_d(l, R) for l in range(7)]
        for l1, l2, l3 in _triples(6):
            C = O.real_cg(l1, l2, l3)
            lhs = np.einsum("ijk,ia,jb->abk", C, D[l1], D[l2])
            rhs = np.einsum("abk,ck->abc", C, D[l3])
            # C(D1 a, D2 b) == D3 C(a, b) for all a, b:
            #   sum_ij C[i,j,k] D1[i,a] D2[j,b] == sum_c D3[k,c] C[a,b,c]
            assert np.allclose(lhs, rhs, atol=1e-10), (l1, l2, l3)


def test_one_one_one_is_cross_product():
    # the only antisymmetric coupling of two vectors: in (y,z,x) order
    # C[a,b,c] = eps / sqrt2 up to the fixed sign
    C = O.real_cg(1, 1, 1)
    a, b = np.array([0.3, -1.2, 0.7]), np.array([1.1, 0.4, -0.5])  # (y,z,x) components
    v = np.einsum("ijk,i,j->k", C, a, b)
    ax, bx = a[[2, 0, 1]], b[[2, 0, 1]]  # to (x,y,z)
    cr = np.cross(ax, bx)[[1, 2, 0]]
    assert np.allclose(np.abs(v), np.abs(cr) / np.sqrt(2), atol=1e-14)
    assert np.allclose(v, cr / np.sqrt(2), atol=1e-14) or np.allclose(v, -cr / np.sqrt(2), atol=1e-14)
