"""The kernel planners' role sets cover the work exactly once (host only).

Read back from the plan's describe() report on every workload (compile-only
plans, no GPU):
  * forward: for each hidden irrep, the roles' channel blocks times their
    path groups cover (channels x paths of the irrep) once, and every role
    sits in one slice;
  * backward: for each hidden irrep with paths, its roles share one phase
    count nph and cover every (32-channel block, edge phase) pair once, all
    in one slice; a slice has no more roles than consumer warps.
The same on irreps sets unlike the workloads, and the one refusal the
planner has (a hidden irrep too wide for shared memory).
"""
import re
from collections import Counter

import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import cgtp as C
from equivariant_mlip_clebsch_b200 import workloads as WL

NAMES = ["tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6", "case4", "case5", "case6"]
# irreps sets unlike the workloads: multiplicities 1, 3, 17, 33 and 96 (partial
# warps and blocks), one irrep without any path, missing outputs, odd parities
ODD = [
    ("3x2o", "1x0e+1x1o", "3x1e+3x2o+3x2e+3x3e"),
    ("1x0e", "1x0e+1x1o+1x2e", "1x1o+1x2e"),
    ("96x1e", "1x0e+1x1o", "96x0o+96x1o"),
    ("128x0e+17x1e+1x2e", "1x0e+1x1o+1x2e", "17x0o+129x0e+35x1e+18x2o+147x2e+1x3o+18x3e+1x4e"),
    ("33x0e", "1x0e+1x1o+1x2e+1x3o+1x4e", "33x0e+33x1o+33x3o+33x4e"),
    ("16x0e+16x1o+8x2e", "1x0e+1x1o", "32x0e+16x1e"),  # 8x2e feeds no output
]


@pytest.fixture
def compile_only(monkeypatch):
    monkeypatch.setenv("CGTP_JIT_COMPILE_ONLY", "1")


def _parse(text, kind):
    head = re.search(rf"^{kind}: roles=(\d+) slices=(\d+) warps=(\d+)\+2", text, re.M)
    nroles, nslices, nw = (int(v) for v in head.groups())
    block = text[head.end():]
    slices = []
    for line in block.splitlines():
        m = re.match(r"\s+slice (\d+):((?: \d+)*)\s*$", line)
        if m:
            slices.append([int(v) for v in m.group(2).split()])
        elif slices and not line.startswith("  slice"):
            break
    return nroles, nw, slices[:nslices]


@pytest.mark.parametrize("irreps", [WL.CONFIGS[n] for n in NAMES] + [
    dict(irreps_in=a, irreps_edge=b, irreps_out=c) for a, b, c in ODD], ids=NAMES + [f"odd{k}" for k in range(len(ODD))])
def test_role_coverage(irreps, compile_only):
    c = irreps
    name = c["irreps_in"]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    text = plan.describe()
    muls = [m for m, _, _ in P.irreps_in]
    npaths = Counter()
    irrep_of_l1 = {}
    for a, (m, l, p) in enumerate(P.irreps_in):
        irrep_of_l1[a] = l
    # path table rows: l1, l2, l3, mul, x_off, k0, o_off, c_off; the hidden
    # irrep of a path is the one whose x block starts at x_off
    x_starts, off = {}, 0
    for a, (m, l, p) in enumerate(P.irreps_in):
        x_starts[off] = a
        off += m * (2 * l + 1)
    for row in P.table:
        npaths[x_starts[int(row[4])]] += 1

    # forward
    nroles, nw, slices = _parse(text, "forward")
    froles = [tuple(int(v) for v in m) for m in
              re.findall(r"frole \d+: irrep (\d+) u0=(\d+) R=(\d+) paths=(\d+)", text)]
    assert len(froles) == nroles
    assert sorted(r for s in slices for r in s) == list(range(nroles))
    assert all(len(s) <= nw for s in slices)
    covered = Counter()
    for a, u0, R, np_ in froles:
        covered[a] += min(32 * R, muls[a] - u0) * np_
    for a in npaths:
        assert covered[a] == muls[a] * npaths[a], (name, a)

    # backward
    nroles, nw, slices = _parse(text, "backward")
    broles = [tuple(int(v) for v in m) for m in
              re.findall(r"brole \d+: irrep (\d+) u0=(\d+) R=(\d+) ph=(\d+)/(\d+)", text)]
    assert len(broles) == nroles
    assert sorted(r for s in slices for r in s) == list(range(nroles))
    assert all(len(s) <= nw for s in slices)
    slice_of = {r: k for k, s in enumerate(slices) for r in s}
    for a in npaths:
        mine = [(i, r) for i, r in enumerate(broles) if r[0] == a]
        assert mine, (name, a)
        assert len({slice_of[i] for i, _ in mine}) == 1  # one slice per irrep
        nph = {r[4] for _, r in mine}
        assert len(nph) == 1
        nph = nph.pop()
        pairs = Counter()
        for _, (_, u0, R, ph, _) in mine:
            for k in range(R):
                if u0 + 32 * k < muls[a]:
                    pairs[(u0 + 32 * k, ph)] += 1
        blocks = range(0, muls[a], 32)
        assert pairs == Counter({(b, ph): 1 for b in blocks for ph in range(nph)}), (name, a)


def test_backward_capacity_refusal(compile_only):
    """One hidden irrep whose grad_out rows do not fit shared memory beside two
    edge stages (256x6e against L = 6 edges: 21 paths, 51,456 floats per atom)
    is refused with CGTP_ERR_SIZE, not planned into an invalid kernel."""
    with pytest.raises(C.CgtpError) as e:
        C.Plan("33x1o+17x4o+256x6e", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o+1x6e",
               "339x1o+340x2o+612x2e+596x3e+613x4o+885x4e+885x5o+852x6o+1091x6e", 6)
    assert e.value.status == 6 and "shared memory" in str(e.value)
