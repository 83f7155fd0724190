"""FP64 CPU oracle of the CGTP convolution (Python side).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference legs of ``bench.py`` are the only callers.  The
product package never imports this module and shares no code with it.

What lives here (the C side is ``cgtp_oracle.c``):
  * irreps-string parsing and path enumeration.  The rule -- every hidden
    irrep (l1,p1) with every edge irrep (l2,p2) and every l3 in
    |l1-l2|..l1+l2 whose (l3, p1*p2) appears in the output irreps -- is the
    reading of LunaTP (arXiv 2610.18393) Table 1 that reproduces all six of its
    output multiplicities (pinned in tests/test_oracle_paths.py);
  * ctypes wrappers around the C loops (CG, SH, neighbour list, forward,
    backward).

Layouts (shared with the product only as a documented interface):
  x   [n_send, D_in]  hidden irrep blocks in order, each [mul, 2l+1]
  Y   [E, (L+1)^2]    degree l at columns l^2 .. l^2+2l, m = -l..l
  W   [E, U]          column = global output channel (output irreps in
                      order, inside a block the paths in enumeration order)
  out [n_recv, D_out] output irrep blocks in order, each [mul, 2l+1]
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cgtp_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liborc.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (FP64, OpenMP, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        d, i, i64 = ctypes.c_double, ctypes.c_int, ctypes.c_int64
        P = ctypes.c_void_p
        L.orc_cg_complex.restype = d
        L.orc_cg_complex.argtypes = [i] * 6
        L.orc_real_cg.restype = i
        L.orc_real_cg.argtypes = [i, i, i, P]
        L.orc_sph_harm.restype = None
        L.orc_sph_harm.argtypes = [i, i64, P, P]
        L.orc_sph_harm_grad.restype = i
        L.orc_sph_harm_grad.argtypes = [i, i64, P, P]
        L.orc_edge_forces.restype = None
        L.orc_edge_forces.argtypes = [i64, P, P, P, P]
        L.orc_edge_virial.restype = None
        L.orc_edge_virial.argtypes = [i64, P, P, P]
        L.orc_neighbor_list.restype = i64
        L.orc_neighbor_list.argtypes = [i64, P, P, d, P, P, P, P]
        L.orc_forward.restype = None
        L.orc_forward.argtypes = [i64, P, P, i, i, i, i, P, P, P, i, P, P, P, i]
        L.orc_backward.restype = None
        L.orc_backward.argtypes = [i64, i64, i64, P, P, i, i, i, i, P, P, P, P, i, P, P,
                                   P, P, P, i]
        L.orc_set_fault.restype = None
        L.orc_set_fault.argtypes = [i]
        L.orc_max_threads.restype = i
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_fault(f: int) -> None:
    """Mutation hook for the tests that check the pins catch planted mistakes."""
    lib().orc_set_fault(int(f))


def max_threads() -> int:
    return int(lib().orc_max_threads())


# ---------------------------------------------------------------------------
# irreps and paths
# ---------------------------------------------------------------------------
_IRREP = re.compile(r"^\s*(\d+)\s*x\s*(\d+)\s*([eo])\s*$")


def parse_irreps(s: str):
    """'128x0e+64x1o' -> [(128, 0, +1), (64, 1, -1)]."""
    out = []
    for tok in s.split("+"):
        m = _IRREP.match(tok)
        if not m:
            raise ValueError(f"cannot parse irrep {tok!r} in {s!r}")
        out.append((int(m.group(1)), int(m.group(2)), 1 if m.group(3) == "e" else -1))
    return out


def dim(irreps) -> int:
    return sum(mul * (2 * l + 1) for mul, l, _ in irreps)


@dataclass
class Paths:
    irreps_in: list
    irreps_edge: list
    irreps_out: list
    L: int
    D_in: int
    D_e: int
    D_out: int
    U: int
    table: np.ndarray  # int32 [P, 8]
    cg: np.ndarray  # float64, concatenated real CG blocks
    out_mul_from_paths: list = field(default_factory=list)

    @property
    def npaths(self) -> int:
        return int(self.table.shape[0])


def enumerate_paths(irreps_in: str, irreps_edge: str, irreps_out: str,
                    check_out: bool = True) -> Paths:
    """Path enumeration and the layout offsets of every path.

    For each hidden irrep (u,l1,p1) in order, each edge irrep (l2,p2) in order
    and each l3 = |l1-l2| .. l1+l2 ascending, the path exists when (l3, p1*p2)
    is one of the output irreps.  Its u channels are appended to that output
    block in this order.  With ``check_out`` the accumulated multiplicity of
    every output block must equal the one declared.
    """
    ii, ie, io = parse_irreps(irreps_in), parse_irreps(irreps_edge), parse_irreps(irreps_out)
    for k, (mul, l, _) in enumerate(ie):
        if mul != 1 or l != k:
            raise ValueError("edge irreps must be 1x0 + 1x1 + ... + 1xL in order")
    L = len(ie) - 1
    keys = [(l, p) for _, l, p in io]
    if len(set(keys)) != len(keys):
        raise ValueError("an (l, parity) appears twice in the output irreps")
    x_off, off = [], 0
    for mul, l, _ in ii:
        x_off.append(off)
        off += mul * (2 * l + 1)
    D_in = off
    out_off, chan_base, off, cb = [], [], 0, 0
    for mul, l, _ in io:
        out_off.append(off)
        chan_base.append(cb)
        off += mul * (2 * l + 1)
        cb += mul
    D_out, U = off, cb
    filled = [0] * len(io)
    rows, blocks, c_off = [], [], 0
    for a, (mul1, l1, p1) in enumerate(ii):
        for (_, l2, p2) in ie:
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                key = (l3, p1 * p2)
                if key not in keys:
                    continue
                o = keys.index(key)
                start = filled[o]
                filled[o] += mul1
                C = real_cg(l1, l2, l3)
                rows.append([l1, l2, l3, mul1, x_off[a], chan_base[o] + start,
                             out_off[o] + start * (2 * l3 + 1), c_off])
                blocks.append(C.ravel())
                c_off += C.size
    if check_out:
        for o, (mul, l, p) in enumerate(io):
            if filled[o] != mul:
                raise ValueError(f"output irrep {mul}x{l}{'e' if p > 0 else 'o'} receives "
                                 f"{filled[o]} channels from the paths")
    table = np.asarray(rows, dtype=np.int32).reshape(-1, 8)
    cg = np.concatenate(blocks) if blocks else np.zeros(0)
    return Paths(ii, ie, io, L, D_in, (L + 1) ** 2, D_out, U, table, cg, filled)


# ---------------------------------------------------------------------------
# coefficient tables and spherical harmonics
# ---------------------------------------------------------------------------
def cg_complex(j1, m1, j2, m2, J, M) -> float:
    return float(lib().orc_cg_complex(j1, m1, j2, m2, J, M))


def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1), dtype=np.float64)
    if lib().orc_real_cg(l1, l2, l3, _ptr(C)) != 0:
        raise ValueError(f"coupling {l1} x {l2} -> {l3} violates the triangle rule")
    return C


def sph_harm(L: int, r) -> np.ndarray:
    r = np.ascontiguousarray(np.asarray(r, dtype=np.float64).reshape(-1, 3))
    Y = np.zeros((r.shape[0], (L + 1) ** 2), dtype=np.float64)
    lib().orc_sph_harm(L, r.shape[0], _ptr(r), _ptr(Y))
    return Y


def sph_harm_grad(L: int, r) -> np.ndarray:
    """Jacobian dY/dr [E, (L+1)^2, 3] of sph_harm, by forward-mode
    differentiation of the same (theta, phi) computation (exact up to
    rounding).  Raises on an edge exactly on the z axis (no derivative of phi)."""
    r = np.ascontiguousarray(np.asarray(r, dtype=np.float64).reshape(-1, 3))
    J = np.zeros((r.shape[0], (L + 1) ** 2, 3), dtype=np.float64)
    if lib().orc_sph_harm_grad(L, r.shape[0], _ptr(r), _ptr(J)) != 0:
        raise ValueError("edge vector on the z axis: the (theta, phi) gradient is undefined there")
    return J


def sph_harm_backward(L: int, r, dY) -> np.ndarray:
    """dL/dr [E, 3] = sum_m dL/dY[e, m] dY_m/dr (the SH step of the force chain)."""
    J = sph_harm_grad(L, r)
    return np.einsum("em,emk->ek", np.asarray(dY, dtype=np.float64), J)


def edge_forces(n_atoms: int, rowptr, col, G) -> np.ndarray:
    """F[a] = -dL/dpos[a] from G = dL/dr per edge (r = pos_sender - pos_receiver + shift)."""
    rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
    col = np.ascontiguousarray(col, dtype=np.int32)
    G = np.ascontiguousarray(G, dtype=np.float64).reshape(-1, 3)
    F = np.zeros((n_atoms, 3), dtype=np.float64)
    lib().orc_edge_forces(int(n_atoms), _ptr(rowptr), _ptr(col), _ptr(G), _ptr(F))
    return F


def edge_virial(r, G) -> np.ndarray:
    """V [3,3] = dL/d strain = sum_e G[e] (outer) r[e], with G = dL/dr per edge
    and every edge vector strained as r -> (1 + eps) r."""
    r = np.ascontiguousarray(r, dtype=np.float64).reshape(-1, 3)
    G = np.ascontiguousarray(G, dtype=np.float64).reshape(-1, 3)
    if r.shape != G.shape:
        raise ValueError("r and G have different edge counts")
    V = np.zeros((3, 3), dtype=np.float64)
    lib().orc_edge_virial(r.shape[0], _ptr(r), _ptr(G), _ptr(V))
    return V


# ---------------------------------------------------------------------------
# neighbour list
# ---------------------------------------------------------------------------
def neighbor_list(pos, box, rc: float):
    """Brute force over all pairs and periodic images.

    Returns (rowptr int64 [N+1], col int32 [E], shift int32 [E,3],
    vec float64 [E,3]) with edges ordered by (receiver, sender, image)."""
    pos = np.ascontiguousarray(pos, dtype=np.float64)
    box = np.ascontiguousarray(box, dtype=np.float64)
    N = pos.shape[0]
    rowptr = np.zeros(N + 1, dtype=np.int64)
    E = lib().orc_neighbor_list(N, _ptr(pos), _ptr(box), float(rc), _ptr(rowptr),
                                None, None, None)
    col = np.zeros(E, dtype=np.int32)
    shift = np.zeros((E, 3), dtype=np.int32)
    vec = np.zeros((E, 3), dtype=np.float64)
    lib().orc_neighbor_list(N, _ptr(pos), _ptr(box), float(rc), _ptr(rowptr), _ptr(col),
                            _ptr(shift), _ptr(vec))
    return rowptr, col, shift, vec


# ---------------------------------------------------------------------------
# the convolution
# ---------------------------------------------------------------------------
def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def forward(paths: Paths, rowptr, col, x, Y, W, nthreads: int = 0) -> np.ndarray:
    rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
    col = np.ascontiguousarray(col, dtype=np.int32)
    x, Y, W = _f64(x), _f64(Y), _f64(W)
    n_recv = rowptr.shape[0] - 1
    out = np.zeros((n_recv, paths.D_out), dtype=np.float64)
    lib().orc_forward(n_recv, _ptr(rowptr), _ptr(col), paths.D_in, paths.D_e, paths.D_out,
                      paths.U, _ptr(x), _ptr(Y), _ptr(W), paths.npaths,
                      _ptr(np.ascontiguousarray(paths.table)), _ptr(paths.cg), _ptr(out),
                      int(nthreads))
    return out


def backward(paths: Paths, rowptr, col, n_send: int, x, Y, W, g, want=("x", "W", "Y"),
             nthreads: int = 0):
    rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
    col = np.ascontiguousarray(col, dtype=np.int32)
    x, Y, W, g = _f64(x), _f64(Y), _f64(W), _f64(g)
    n_recv = rowptr.shape[0] - 1
    E = col.shape[0]
    dx = np.zeros((n_send, paths.D_in)) if "x" in want else None
    dW = np.zeros((E, paths.U)) if "W" in want else None
    dY = np.zeros((E, paths.D_e)) if "Y" in want else None
    lib().orc_backward(n_recv, n_send, E, _ptr(rowptr), _ptr(col), paths.D_in, paths.D_e,
                       paths.D_out, paths.U, _ptr(x), _ptr(Y), _ptr(W), _ptr(g), paths.npaths,
                       _ptr(np.ascontiguousarray(paths.table)), _ptr(paths.cg), _ptr(dx),
                       _ptr(dW), _ptr(dY), int(nthreads))
    return dx, dW, dY


def double_backward(paths: Paths, rowptr, col, n_send: int, x, Y, W, g, h_x=None, h_W=None, h_Y=None):
    """Gradients of S = <h_x, dx> + <h_W, dW> + <h_Y, dY>, (dx, dW, dY) the
    backward of the convolution at (x, Y, W) with cotangent g, with respect
    to g, x, W and Y (None cotangents are zero).  The convolution is linear
    in each of x, Y and W, so each term of S is the pairing of g with a
    forward in which one argument is replaced by its cotangent:
        S = <g, fwd(h_x, Y, W) + fwd(x, Y, h_W) + fwd(x, h_Y, W)>
    and every gradient is a forward or a backward with that substitution.
    Written as those calls of forward() and backward() above."""
    n_recv = len(rowptr) - 1
    E = len(col)
    gg = np.zeros((n_recv, paths.D_out))
    gx = np.zeros((n_send, paths.D_in))
    gW = np.zeros((E, paths.U))
    gY = np.zeros((E, paths.D_e))
    if h_x is not None:  # <g, fwd(h_x, Y, W)>: depends on g, Y, W
        gg += forward(paths, rowptr, col, h_x, Y, W)
        _, dW, dY = backward(paths, rowptr, col, n_send, h_x, Y, W, g, want=("W", "Y"))
        gW += dW
        gY += dY
    if h_W is not None:  # <g, fwd(x, Y, h_W)>: depends on g, x, Y
        gg += forward(paths, rowptr, col, x, Y, h_W)
        dx, _, dY = backward(paths, rowptr, col, n_send, x, Y, h_W, g, want=("x", "Y"))
        gx += dx
        gY += dY
    if h_Y is not None:  # <g, fwd(x, h_Y, W)>: depends on g, x, W
        gg += forward(paths, rowptr, col, x, h_Y, W)
        dx, dW, _ = backward(paths, rowptr, col, n_send, x, h_Y, W, g, want=("x", "W"))
        gx += dx
        gW += dW
    return gg, gx, gW, gY


# ---------------------------------------------------------------------------
# BranchIP sparse evaluation (BranchIP page, section "BranchIP" and the
# Branchlegro paragraph): a router gives every edge a continuation gate
# f_e in [0, 1]; the gate multiplies the edge's feature before the TP, so the
# edge's TP term is scaled by f_e (the convolution is linear in W, so the gate
# is applied to the edge's weight row here).  Dense evaluation keeps every
# edge; sparse evaluation omits the zero-gated edges from the TP and pads the
# skipped per-edge outputs with zeros over the full edge set.
# ---------------------------------------------------------------------------
def gated_forward(paths: Paths, rowptr, col, x, Y, W, gate) -> np.ndarray:
    """Dense evaluation: every edge, its TP term scaled by its gate."""
    gate = np.asarray(gate, dtype=np.float64)
    return forward(paths, rowptr, col, x, Y, gate[:, None] * _f64(W))


def gated_backward(paths: Paths, rowptr, col, n_send: int, x, Y, W, gate, g):
    """Gradients of <g, gated_forward> with respect to x, W, Y and the gate,
    every edge evaluated (dense).  With W' = gate * W: dW = gate * dL/dW',
    dgate[e] = <W[e], dL/dW'[e]> (= <g[i], the edge's ungated TP term>)."""
    gate = np.asarray(gate, dtype=np.float64)
    W = _f64(W)
    dx, dWp, dY = backward(paths, rowptr, col, n_send, x, Y, gate[:, None] * W, g)
    return dx, gate[:, None] * dWp, dY, np.sum(W * dWp, axis=1)


def active_edges(rowptr, gate):
    """The sparse evaluation's edge set: the edges with a non-zero gate, in
    their original (receiver-sorted) order, and the receiver CSR over them.
    Returns (act int64 [E_A] edge ids, rowptr_A int64 [n_recv+1])."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    gate = np.asarray(gate, dtype=np.float64)
    n_recv = len(rowptr) - 1
    recv = np.repeat(np.arange(n_recv), np.diff(rowptr))
    act = np.nonzero(gate > 0)[0]
    rowptr_A = np.concatenate([[0], np.cumsum(np.bincount(recv[act], minlength=n_recv))]).astype(np.int64)
    return act, rowptr_A


def sparse_forward(paths: Paths, rowptr, col, x, Y, W, gate) -> np.ndarray:
    """Sparse evaluation: the TP runs on the active edges only."""
    gate = np.asarray(gate, dtype=np.float64)
    act, rowptr_A = active_edges(rowptr, gate)
    col = np.asarray(col)
    return forward(paths, rowptr_A, col[act], x, _f64(Y)[act], gate[act, None] * _f64(W)[act])


def sparse_backward(paths: Paths, rowptr, col, n_send: int, x, Y, W, gate, g):
    """Sparse evaluation of the gradients: the backward runs on the active
    edges only, and dW, dY and dgate of the skipped edges are zero (no
    backward branch is built for them).  dx, dW and dY equal the dense ones
    exactly (a zero gate scales the skipped edges' terms to zero); dgate
    equals the dense one on active edges and is zero on skipped ones, which
    is exact for any loss reaching the gate through a function with zero
    slope wherever it is zero (the pages' flat-zero gate)."""
    gate = np.asarray(gate, dtype=np.float64)
    W, Y = _f64(W), _f64(Y)
    act, rowptr_A = active_edges(rowptr, gate)
    col = np.asarray(col)
    E = len(col)
    dx, dWp, dYa = backward(paths, rowptr_A, col[act], n_send, x, Y[act], gate[act, None] * W[act], g)
    dW = np.zeros((E, paths.U))
    dY = np.zeros((E, paths.D_e))
    dgate = np.zeros(E)
    dW[act] = gate[act, None] * dWp
    dY[act] = dYa
    dgate[act] = np.sum(W[act] * dWp, axis=1)
    return dx, dW, dY, dgate
