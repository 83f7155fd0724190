"""Pins of the oracle's periodic neighbour list.

Silicon in the diamond structure (a = 5.43 A, the MD system of the LunaTP
page, Fig. 6) has neighbour shells at a*sqrt3/4, a/sqrt2, a*sqrt11/4, a and
a*sqrt19/4 holding 4, 12, 12, 6 and 12 atoms.  A perfect crystal therefore has
exactly 28 neighbours within 5.0 A and 46 within 6.0 A -- whatever the size
of the periodic box, as long as every periodic image is counted.
"""
import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200.workloads import SI_A, si_diamond


def test_shell_radii_bracket_the_cutoffs():
    shells = SI_A * np.array([np.sqrt(3) / 4, 1 / np.sqrt(2), np.sqrt(11) / 4, 1.0, np.sqrt(19) / 4])
    assert shells[2] < 5.0 < shells[3] and shells[4] < 6.0


@pytest.mark.parametrize("cells,rc,deg", [((2, 2, 2), 5.0, 28), ((2, 2, 2), 6.0, 46),
                                          ((1, 1, 1), 5.0, 28), ((1, 1, 2), 6.0, 46),
                                          ((3, 2, 2), 5.0, 28)])
def test_perfect_lattice_coordination(cells, rc, deg):
    pos, box = si_diamond(cells, sigma=0.0)
    rowptr, col, shift, vec = O.neighbor_list(pos, box, rc)
    assert np.all(np.diff(rowptr) == deg)


def test_edges_symmetric_and_vectors_consistent():
    pos, box = si_diamond((2, 2, 2), sigma=0.05, seed=0)
    rowptr, col, shift, vec = O.neighbor_list(pos, box, 5.0)
    recv = np.repeat(np.arange(len(pos)), np.diff(rowptr))
    d = pos[col] + shift * box - pos[recv]
    assert np.array_equal(d, vec)
    assert np.all((vec ** 2).sum(1) < 25.0)
    fwd = set(zip(recv.tolist(), col.tolist(), map(tuple, shift.tolist())))
    rev = set(zip(col.tolist(), recv.tolist(), map(tuple, (-shift).tolist())))
    assert fwd == rev
    # sorted by (receiver, sender, image)
    key = np.lexsort((shift[:, 2], shift[:, 1], shift[:, 0], col, recv))
    assert np.array_equal(key, np.arange(len(col)))


def test_self_pair_excluded_and_self_images_kept():
    # one atom in a 4 A cube: its own images at 4 A are neighbours within 5 A
    rowptr, col, shift, vec = O.neighbor_list(np.zeros((1, 3)), np.array([4.0, 4.0, 4.0]), 5.0)
    assert rowptr[1] == 6
    assert set(map(tuple, shift.tolist())) == {(1, 0, 0), (-1, 0, 0), (0, 1, 0), (0, -1, 0),
                                               (0, 0, 1), (0, 0, -1)}
