"""Seeded workload construction shared by the parity tests.

Inputs come from equivariant_mlip_clebsch_b200.workloads (positions and random
draws only).  The expected side (CSR, edge vectors, path table, per-column W
scale) is computed by the oracle; the CUDA side computes its own CSR and edge
vectors and is checked against the oracle's bit for bit before use.
"""
import numpy as np

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL


def oracle_fan_in(P: "O.Paths"):
    """Number of paths feeding each output irrep block (from the oracle)."""
    bases = np.concatenate([[0], np.cumsum([m for m, _, _ in P.irreps_out])])
    fan = np.zeros(len(P.irreps_out), dtype=int)
    for k0 in P.table[:, 5]:
        fan[np.searchsorted(bases, k0, side="right") - 1] += 1
    return fan


class Workload:
    """Oracle view of one synthetic workload."""

    def __init__(self, name: str, seed: int = 0):
        c = WL.CONFIGS[name]
        self.name, self.cfg = name, c
        self.pos, self.box = WL.si_diamond(c["cells"], c["sigma"], seed)
        self.rowptr, self.col, self.shift, self.vec = O.neighbor_list(self.pos, self.box, c["rc"])
        self.r32 = self.vec.astype(np.float32)
        self.P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
        self.N, self.E = len(self.pos), len(self.col)
        muls = [m for m, _, _ in self.P.irreps_out]
        self.col_std = WL.column_std(muls, oracle_fan_in(self.P))
        self.x = WL.draw_x(self.N, self.P.D_in, seed)
        self.W = WL.draw_W(self.E, self.P.U, self.col_std, seed)
        self.g = WL.draw_g(self.N, self.P.D_out, seed)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close(got, ref, what: str, rel=1e-5, maxfrac=1e-4):
    """rel-L2 <= 1e-5 and max |err| <= 1e-4 * max |ref| (the acceptance bar)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if ref.size == 0:
        return
    r = rel_l2(got, ref)
    m = float(np.abs(got - ref).max())
    scale = float(np.abs(ref).max())
    assert r <= rel and m <= maxfrac * max(scale, 1e-30), \
        f"{what}: rel-L2 {r:.3e} (bar {rel}), max err {m:.3e} vs {maxfrac} x {scale:.3e}"
