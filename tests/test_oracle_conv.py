"""Pins of the oracle's CGTP forward and backward.

The operation (LunaTP, arXiv 2610.18393, Abstract; outputs x' and gradients
x-bar, y-bar, w-bar of Table 11), read plainly:
  out[i] = sum_{e: i<-j} sum_paths W[e, path, u] CG(x_j[u], Y(r_e))
Pins, none of which re-types the oracle's loops:
  * a dense Kronecker-product contraction on tiny graphs (a different
    organisation of the same sum: one sparse matrix per edge applied to
    vec(x_j (x) Y_e));
  * equivariance, f(phi(g) x) = rho(g) f(x) (TransIP page, Sec. 2.1, Eq. 1),
    with Wigner-D matrices, to 1e-10 in FP64; inversion for natural parity;
  * special cases: a single 0e x 0e -> 0e path is a weighted sparse
    matrix-vector sum; the 0 x l -> l paths carry Y_l(r) times x_j;
  * sparse evaluation equals dense evaluation with zero-weight edges
    (BranchIP page, Sec. "BranchIP": a TP with a zero-gated input vanishes);
  * backward: the trilinear identity <g,out> = <dx,x> = <dW,W> = <dY,Y>,
    central finite differences, and equivariance of the gradients;
  * planted mistakes in the oracle (dropped terms, a sign flip in the real
    basis) make these pins fail.
"""
import numpy as np
import pytest
import scipy.sparse as sp

import oracle as O
from equivariant_mlip_clebsch_b200.workloads import CONFIGS
from tests._so3 import block_rotation, random_rotation


def shrink(name, mul):
    """Irreps of a workload with every hidden multiplicity set to ``mul``."""
    c = CONFIGS[name]
    hid = "+".join(f"{mul}x{l}{'e' if p > 0 else 'o'}" for _, l, p in O.parse_irreps(c["irreps_in"]))
    P0 = O.enumerate_paths(hid, c["irreps_edge"], c["irreps_out"], check_out=False)
    out = "+".join(f"{m}x{l}{'e' if p > 0 else 'o'}"
                   for m, (_, l, p) in zip(P0.out_mul_from_paths, P0.irreps_out) if m > 0)
    return hid, c["irreps_edge"], out


def random_graph(rng, n_recv, n_send, max_deg=5, allow_empty=True):
    deg = rng.integers(0 if allow_empty else 1, max_deg + 1, size=n_recv)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    col = rng.integers(0, n_send, size=rowptr[-1]).astype(np.int32)
    r = rng.standard_normal((rowptr[-1], 3)) * 2.0
    return rowptr, col, r


def problem(irreps, n=6, seed=0, max_deg=5):
    rng = np.random.default_rng(seed)
    P = O.enumerate_paths(*irreps)
    rowptr, col, r = random_graph(rng, n, n, max_deg)
    E = len(col)
    x = rng.standard_normal((n, P.D_in))
    W = rng.standard_normal((E, P.U))
    g = rng.standard_normal((n, P.D_out))
    return P, rowptr, col, r, x, W, g


def dense_kronecker_forward(P, rowptr, col, x, Y, W):
    rows, cols, vals, wcol = [], [], [], []
    off = 0
    for (l1, l2, l3, mul, xo, k0, oo, co) in P.table:
        n1, n2, n3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
        C = P.cg[co:co + n1 * n2 * n3].reshape(n1, n2, n3)
        a, b, c = np.nonzero(C)
        for u in range(mul):
            rows.append(oo + u * n3 + c)
            cols.append((xo + u * n1 + a) * P.D_e + l2 * l2 + b)
            vals.append(C[a, b, c])
            wcol.append(np.full(len(a), k0 + u))
    rows, cols, vals, wcol = map(np.concatenate, (rows, cols, vals, wcol))
    out = np.zeros((len(rowptr) - 1, P.D_out))
    for i in range(len(rowptr) - 1):
        for e in range(rowptr[i], rowptr[i + 1]):
            M = sp.coo_matrix((vals * W[e, wcol], (rows, cols)), shape=(P.D_out, P.D_in * P.D_e))
            out[i] += M @ np.kron(x[col[e]], Y[e])
    return out


CASES = ["tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6"]
NATURAL = ["tiny", "lmax2_wide", "lmax3", "lmax6"]  # edge labels equal (-1)^l


@pytest.mark.parametrize("name", CASES)
def test_dense_kronecker(name):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 2), n=5, max_deg=3)
    Y = O.sph_harm(P.L, r)
    out = O.forward(P, rowptr, col, x, Y, W)
    ref = dense_kronecker_forward(P, rowptr, col, x, Y, W)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def _equivariance_error(P, rowptr, col, r, x, W, R, parity=1):
    Din = block_rotation(P.irreps_in, R, parity)
    Dout = block_rotation(P.irreps_out, R, parity)
    Rr = parity * (r @ R.T)
    out = O.forward(P, rowptr, col, x, O.sph_harm(P.L, r), W)
    out_rot = O.forward(P, rowptr, col, x @ Din.T, O.sph_harm(P.L, Rr), W)
    return np.abs(out_rot - out @ Dout.T).max() / max(np.abs(out).max(), 1.0)


@pytest.mark.parametrize("name", CASES)
def test_forward_equivariance(name):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 3), n=6)
    R = random_rotation(np.random.default_rng(21))
    assert _equivariance_error(P, rowptr, col, r, x, W, R) < 1e-10


@pytest.mark.parametrize("name", NATURAL)
def test_forward_inversion(name):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 2), n=6)
    R = random_rotation(np.random.default_rng(22))
    assert _equivariance_error(P, rowptr, col, r, x, W, R, parity=-1) < 1e-10


def test_scalar_path_is_weighted_spmv():
    P, rowptr, col, r, x, W, g = problem(("4x0e", "1x0e", "4x0e"), n=7)
    out = O.forward(P, rowptr, col, x, O.sph_harm(0, r), W)
    ref = np.zeros_like(out)
    recv = np.repeat(np.arange(7), np.diff(rowptr))
    np.add.at(ref, recv, W * x[col])
    assert np.allclose(out, ref, atol=1e-13)


def test_zero_to_l_paths_carry_the_harmonics():
    P, rowptr, col, r, x, W, g = problem(("3x0e", "1x0e+1x1o+1x2e", "3x0e+3x1o+3x2e"), n=6)
    Y = O.sph_harm(2, r)
    out = O.forward(P, rowptr, col, x, Y, W)
    recv = np.repeat(np.arange(6), np.diff(rowptr))
    for l in range(3):
        ref = np.zeros((6, 3, 2 * l + 1))
        msg = (W[:, 3 * l:3 * l + 3] * x[col])[:, :, None] * Y[:, None, l * l:(l + 1) ** 2]
        np.add.at(ref, recv, msg)
        o = 3 * (l * l)
        assert np.allclose(out[:, o:o + 3 * (2 * l + 1)], ref.reshape(6, -1), atol=1e-13)


def test_sparse_equals_dense_with_zero_weights():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax3", 2), n=8, max_deg=6)
    Y = O.sph_harm(P.L, r)
    rng = np.random.default_rng(3)
    keep = rng.random(len(col)) < 0.5
    Wd = W.copy()
    Wd[~keep] = 0.0
    dense = O.forward(P, rowptr, col, x, Y, Wd)
    recv = np.repeat(np.arange(8), np.diff(rowptr))
    rp = np.concatenate([[0], np.cumsum(np.bincount(recv[keep], minlength=8))]).astype(np.int64)
    sparse = O.forward(P, rp, col[keep], x, Y[keep], W[keep])
    assert np.array_equal(dense, sparse)


def test_empty_graph_and_empty_rows():
    P = O.enumerate_paths("4x0e+2x1o", "1x0e+1x1o", "6x0e+6x1o")
    out = O.forward(P, np.zeros(4, np.int64), np.zeros(0, np.int32), np.ones((3, P.D_in)),
                    np.zeros((0, 4)), np.zeros((0, P.U)))
    assert out.shape == (3, P.D_out) and np.all(out == 0)


@pytest.mark.parametrize("name", CASES)
def test_backward_trilinear_identity(name):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 2), n=6)
    Y = O.sph_harm(P.L, r)
    out = O.forward(P, rowptr, col, x, Y, W)
    dx, dW, dY = O.backward(P, rowptr, col, 6, x, Y, W, g)
    s = (g * out).sum()
    for grad, val in ((dx, x), (dW, W), (dY, Y)):
        assert (grad * val).sum() == pytest.approx(s, rel=1e-11, abs=1e-11)


def test_backward_finite_differences():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax3", 2), n=5)
    Y = O.sph_harm(P.L, r)
    dx, dW, dY = O.backward(P, rowptr, col, 5, x, Y, W, g)
    loss = lambda x_, Y_, W_: (g * O.forward(P, rowptr, col, x_, Y_, W_)).sum()
    rng = np.random.default_rng(9)
    h = 1e-3
    for arr, grad, which in ((x, dx, 0), (Y, dY, 1), (W, dW, 2)):
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            args_p = [x, Y, W]
            args_m = [x, Y, W]
            args_p[which], args_m[which] = ap, am
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert fd == pytest.approx(grad[idx], rel=1e-7, abs=1e-9)


def test_backward_equivariance():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax3", 2), n=6)
    R = random_rotation(np.random.default_rng(23))
    Din = block_rotation(P.irreps_in, R)
    Dout = block_rotation(P.irreps_out, R)
    De = block_rotation(P.irreps_edge, R)
    Y, YR = O.sph_harm(P.L, r), O.sph_harm(P.L, r @ R.T)
    dx, dW, dY = O.backward(P, rowptr, col, 6, x, Y, W, g)
    dxR, dWR, dYR = O.backward(P, rowptr, col, 6, x @ Din.T, YR, W, g @ Dout.T)
    assert np.allclose(dxR, dx @ Din.T, atol=1e-10)
    assert np.allclose(dYR, dY @ De.T, atol=1e-10)
    assert np.allclose(dWR, dW, atol=1e-10)


def test_pins_catch_planted_mistakes():
    try:
        O.set_fault(1)  # forward drops every m2 > 0 term
        P, rowptr, col, r, x, W, g = problem(shrink("lmax2", 2), n=5, max_deg=3)
        Y = O.sph_harm(P.L, r)
        assert not np.allclose(O.forward(P, rowptr, col, x, Y, W),
                               dense_kronecker_forward(P, rowptr, col, x, Y, W), atol=1e-8)
        O.set_fault(2)  # real basis of the CG tables without the (-1)^m of the m>0 rows
        P, rowptr, col, r, x, W, g = problem(shrink("lmax3", 2), n=6)
        R = random_rotation(np.random.default_rng(21))
        assert _equivariance_error(P, rowptr, col, r, x, W, R) > 1e-3
    finally:
        O.set_fault(0)
