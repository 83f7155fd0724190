"""Pins of the oracle's path enumeration and layout offsets.

LunaTP (arXiv 2610.18393) Appendix Table 1 prints, for six irreps
configurations, the output multiplicities the CGTP produces.  The
enumeration rule (every hidden irrep x every edge irrep x every l3 in the
triangle whose (l3, p1 p2) is an output irrep, each path adding mul(l1)
channels) must reproduce every one of them.
"""
import os

import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200.workloads import CONFIGS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lunatp_table1.txt")


def _table1():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        case, lmax, hid, edge, out = [t.strip() for t in line.split("|")]
        rows.append((int(case), int(lmax), hid.replace(" ", ""), edge.replace(" ", ""),
                     out.replace(" ", "")))
    return rows


@pytest.mark.parametrize("row", _table1(), ids=lambda r: f"case{r[0]}")
def test_table1_output_multiplicities(row):
    _, lmax, hid, edge, out = row
    P = O.enumerate_paths(hid, edge, out, check_out=False)
    declared = [mul for mul, _, _ in O.parse_irreps(out)]
    assert P.out_mul_from_paths == declared
    assert P.L == lmax or P.L == lmax + 1  # Case 2 and 3 edges reach l=3
    # a consistent plan must accept it with the check on
    O.enumerate_paths(hid, edge, out, check_out=True)


@pytest.mark.parametrize("name,npaths", [("tiny", 4), ("lmax2", 15), ("lmax2_wide", 17),
                                         ("lmax3", 23), ("lmax6", 106)])
def test_path_counts_of_workloads(name, npaths):
    c = CONFIGS[name]
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    assert P.npaths == npaths
    assert P.U == sum(P.out_mul_from_paths)


def test_layout_offsets_cover_output_exactly():
    c = CONFIGS["lmax3"]
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    cover = np.zeros(P.D_out, dtype=int)
    wcov = np.zeros(P.U, dtype=int)
    for l1, l2, l3, mul, xo, k0, oo, co in P.table:
        cover[oo:oo + mul * (2 * l3 + 1)] += 1
        wcov[k0:k0 + mul] += 1
        assert xo + mul * (2 * l1 + 1) <= P.D_in
    assert np.all(cover == 1) and np.all(wcov == 1)


def test_mismatched_output_rejected():
    with pytest.raises(ValueError):
        O.enumerate_paths("16x0e+16x1o", "1x0e+1x1o", "32x0e+16x1o")
    with pytest.raises(ValueError):
        O.enumerate_paths("16x0e", "1x0e+1x2e", "16x0e")  # edge must be 0..L
    with pytest.raises(ValueError):
        O.parse_irreps("16x0e+4y1o")
