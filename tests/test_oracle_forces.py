"""Pins of the oracle's force chain: dL/dY -> dL/dr (SH gradient) -> forces.

Forces are minus the position gradient of the energy (the BranchIP page's
force definition); the CGTP backward's dL/dY feeds them through the gradient
of the spherical harmonics with respect to the edge vector.  The oracle takes
that gradient by forward-mode differentiation of its own (theta, phi)
harmonics; these tests pin it to things other than itself:
  * closed forms: Y_1 = sqrt3 (y, z, x)/r and Y_2,-2 = sqrt15 x y / r^2,
  * Y depends on the direction only: r . dY/dr = 0, dY/dr(s r) = dY/dr(r)/s,
  * central finite differences of the oracle's harmonics,
  * rotation: dY/dr(R r) = D(R) dY/dr(r) R^T,
  * forces: they sum to zero, and equal minus the finite-difference position
    gradient of an energy built from the harmonics on a periodic cell,
  * the virial (strain derivative): it equals the finite-difference strain
    derivative of such an energy (with a radial factor, so the isotropic part
    counts), and its trace vanishes for an energy of the directions alone,
  * planted mistakes (the phi term dropped, a sign flipped in the force
    assembly, the virial transposed) fail these pins.
"""
import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL
from tests._so3 import random_rotation, wigner_d


def _vectors(n, seed):
    r = np.random.default_rng(seed).standard_normal((n, 3))
    return r * np.random.default_rng(seed + 1).uniform(0.5, 3.0, size=(n, 1))


def test_l1_closed_form():
    r = _vectors(50, 1)
    J = O.sph_harm_grad(1, r)
    n = np.linalg.norm(r, axis=1)
    u = r / n[:, None]
    # Y_1 = sqrt3 (u_y, u_z, u_x); d u_a / d r_k = (delta_ak - u_a u_k) / |r|
    for comp, a in ((1, 1), (2, 2), (3, 0)):
        ref = np.sqrt(3.0) * ((np.arange(3) == a)[None, :] - u[:, a:a + 1] * u) / n[:, None]
        assert np.allclose(J[:, comp, :], ref, atol=1e-13)
    assert np.allclose(J[:, 0, :], 0.0)


def test_l2_closed_form():
    r = _vectors(50, 2)
    x, y, z = r.T
    r2 = (r * r).sum(1)
    Y = O.sph_harm(2, r)
    assert np.allclose(Y[:, 4], np.sqrt(15.0) * x * y / r2, atol=1e-13)
    J = O.sph_harm_grad(2, r)
    ref = np.sqrt(15.0) * (np.stack([y, x, 0 * z], 1) / r2[:, None] - 2 * (x * y)[:, None] * r / (r2 * r2)[:, None])
    assert np.allclose(J[:, 4, :], ref, atol=1e-12)


@pytest.mark.parametrize("L", [3, 6])
def test_direction_only(L):
    r = _vectors(40, 3 + L)
    J = O.sph_harm_grad(L, r)
    assert np.abs(np.einsum("ek,etk->et", r, J)).max() < 1e-11 * np.abs(J).max()
    J2 = O.sph_harm_grad(L, 2.5 * r)
    assert np.allclose(J2, J / 2.5, atol=1e-12)


@pytest.mark.parametrize("L", [2, 6])
def test_finite_differences(L):
    r = _vectors(30, 11 + L)
    J = O.sph_harm_grad(L, r)
    h = 1e-5
    for k in range(3):
        rp, rm = r.copy(), r.copy()
        rp[:, k] += h
        rm[:, k] -= h
        fd = (O.sph_harm(L, rp) - O.sph_harm(L, rm)) / (2 * h)
        assert np.abs(fd - J[:, :, k]).max() < 1e-7 * max(1.0, np.abs(J).max())


def test_rotation():
    L = 4
    r = _vectors(30, 21)
    R = random_rotation(np.random.default_rng(22))
    J, JR = O.sph_harm_grad(L, r), O.sph_harm_grad(L, r @ R.T)
    for l in range(L + 1):
        D = wigner_d(l, R)
        sl = slice(l * l, (l + 1) * (l + 1))
        ref = np.einsum("ab,ebk,jk->eaj", D, J[:, sl, :], R)
        assert np.allclose(JR[:, sl, :], ref, atol=1e-8)


def test_zero_vector_and_axis():
    assert np.all(O.sph_harm_grad(3, np.zeros((1, 3))) == 0.0)
    with pytest.raises(ValueError):
        O.sph_harm_grad(3, np.array([[0.0, 0.0, 1.0]]))


def _cell_energy_and_forces(seed=0, L=2, h=1e-5, fault=0):
    """E(pos) = sum_e sum_m c[e,m] Y_m(r_e(pos)) on the tiny Si cell with its
    edge list (and image shifts) held fixed; forces by the oracle chain and by
    central differences of E over the positions."""
    c = WL.CONFIGS["tiny"]
    pos, box = WL.si_diamond(c["cells"], c["sigma"], seed)
    rowptr, col, shift, vec = O.neighbor_list(pos, box, c["rc"])
    recv = np.repeat(np.arange(len(pos)), np.diff(rowptr))
    coef = np.random.default_rng(seed + 5).standard_normal((len(col), (L + 1) ** 2))

    def edges(p):
        return p[col] + shift * box[None, :] - p[recv]

    assert np.allclose(edges(pos), vec, atol=1e-12)

    def energy(p):
        return float((coef * O.sph_harm(L, edges(p))).sum())

    try:
        O.set_fault(fault)
        F = O.edge_forces(len(pos), rowptr, col, O.sph_harm_backward(L, vec, coef))
    finally:
        O.set_fault(0)
    sel = [(a, k) for a in (0, 3, 17, 40) for k in range(3)]
    fd = []
    for a, k in sel:
        pp, pm = pos.copy(), pos.copy()
        pp[a, k] += h
        pm[a, k] -= h
        fd.append(-(energy(pp) - energy(pm)) / (2 * h))
    return F, np.array([F[a, k] for a, k in sel]), np.array(fd)


def test_forces_against_energy_differences():
    F, got, fd = _cell_energy_and_forces()
    assert np.abs(F.sum(0)).max() < 1e-9 * np.abs(F).max()  # no net force
    assert np.abs(got - fd).max() < 1e-6 * max(1.0, np.abs(fd).max())


def test_pins_catch_planted_mistakes():
    try:
        O.set_fault(3)  # the phi term of the gradient dropped
        r = _vectors(20, 31)
        J = O.sph_harm_grad(2, r)
    finally:
        O.set_fault(0)
    h = 1e-5
    rp, rm = r.copy(), r.copy()
    rp[:, 0] += h
    rm[:, 0] -= h
    fd = (O.sph_harm(2, rp) - O.sph_harm(2, rm)) / (2 * h)
    assert np.abs(fd - J[:, :, 0]).max() > 1e-3
    F, got, fd = _cell_energy_and_forces(fault=4)  # sign of the sender term flipped
    assert np.abs(got - fd).max() > 1e-3


def _strained_energy_and_virial(seed=0, L=3, h=1e-6, fault=0):
    """E(eps) = sum_e |r_e|^2 sum_m c[e,m] Y_m(r_e) over the tiny Si cell's
    edges with every edge vector strained, r_e -> (1 + eps) r_e (edge list and
    images held fixed).  Returns the oracle's virial of G = dE/dr and the
    central differences of E over the nine strain components."""
    c = WL.CONFIGS["tiny"]
    pos, box = WL.si_diamond(c["cells"], c["sigma"], seed)
    _, col, _, vec = O.neighbor_list(pos, box, c["rc"])
    coef = np.random.default_rng(seed + 9).standard_normal((len(col), (L + 1) ** 2))

    def energy(eps):
        r = vec @ (np.eye(3) + eps).T
        return float(((r * r).sum(1)[:, None] * coef * O.sph_harm(L, r)).sum())

    # dE/dr_e = |r|^2 sum_m c dY_m/dr + 2 r sum_m c Y_m (product rule)
    s = (coef * O.sph_harm(L, vec)).sum(1)
    G = (vec * vec).sum(1)[:, None] * O.sph_harm_backward(L, vec, coef) + 2.0 * vec * s[:, None]
    try:
        O.set_fault(fault)
        V = O.edge_virial(vec, G)
    finally:
        O.set_fault(0)
    fd = np.zeros((3, 3))
    for a in range(3):
        for b in range(3):
            d = np.zeros((3, 3))
            d[a, b] = h
            fd[a, b] = (energy(d) - energy(-d)) / (2 * h)
    return V, fd


def test_virial_against_strain_differences():
    V, fd = _strained_energy_and_virial()
    assert np.abs(V - V.T).max() > 1e-2 * np.abs(V).max()  # asymmetric: a transposition shows
    assert abs(np.trace(V)) > 1e-2 * np.abs(V).max()      # the isotropic part is exercised
    assert np.abs(V - fd).max() < 1e-6 * np.abs(fd).max()


def test_virial_trace_vanishes_for_directions_only():
    """Y depends on the direction alone, so a uniform dilation leaves an
    energy of the harmonics unchanged: sum_e G_e . r_e = trace V = 0."""
    r = _vectors(200, 41)
    coef = np.random.default_rng(42).standard_normal((200, 16))
    V = O.edge_virial(r, O.sph_harm_backward(3, r, coef))
    assert abs(np.trace(V)) < 1e-12 * np.abs(V).sum()
    assert np.abs(V).max() > 1.0


def test_virial_pin_catches_transposition():
    V, fd = _strained_energy_and_virial(fault=5)
    assert np.abs(V - fd).max() > 1e-2 * np.abs(fd).max()
