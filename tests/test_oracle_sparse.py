"""Pins of the oracle's BranchIP sparse evaluation.

The BranchIP page (section "BranchIP", the Branchlegro paragraph) gives every
edge a continuation gate f_e in [0, 1] that multiplies the edge's feature
before the TP; at inference the zero-gated edges are omitted from the TP and
the skipped per-edge outputs are zero-padded to the full edge set, and the
page states that this sparse path reproduces the dense evaluation exactly,
derivatives included, when the gate is identically zero (with zero slope)
around every removed edge.  Pins, none of which re-types the oracle's code:
  * sparse == dense (out, dx, dW, dY to FP64 rounding; the gate gradient on
    the active edges), on several irreps sets with a third to all of the
    gates zero;
  * all gates one: the ungated convolution; all gates zero: zeros;
  * the gate gradient is the derivative of S = <g, out> in each gate, by a
    finite difference (S is linear in every gate, so the difference is exact
    up to rounding), on active and on skipped edges (where the dense
    derivative is not zero, and the sparse path reports zero);
  * through a flat-zero C2 gate function f = F(nu) (a clamped quintic
    smoothstep, a test tool: the page gives F's properties, not its formula),
    the sparse chain dS/dnu = dgate * F'(nu) equals the finite difference of
    S(F(nu)) on every edge, the skipped ones included;
  * a planted mistake (a wrong activity threshold) fails the first pin.
"""
import numpy as np
import pytest

import oracle as O
from tests.test_oracle_conv import problem, shrink


def gates(rng, E, frac_zero):
    f = rng.uniform(0.05, 1.0, size=E)
    f[rng.uniform(size=E) < frac_zero] = 0.0
    return f


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("name,frac", [("tiny", 0.5), ("lmax2", 0.3), ("lmax2_wide", 0.7), ("lmax3", 1.0)])
def test_sparse_equals_dense(name, frac):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 3), n=7, seed=11)
    rng = np.random.default_rng(5)
    Y = O.sph_harm(P.L, r)
    f = gates(rng, len(col), frac)
    out_s = O.sparse_forward(P, rowptr, col, x, Y, W, f)
    out_d = O.gated_forward(P, rowptr, col, x, Y, W, f)
    assert rel(out_s, out_d) < 1e-13
    dx_s, dW_s, dY_s, df_s = O.sparse_backward(P, rowptr, col, len(x), x, Y, W, f, g)
    dx_d, dW_d, dY_d, df_d = O.gated_backward(P, rowptr, col, len(x), x, Y, W, f, g)
    on = f > 0
    assert rel(dx_s, dx_d) < 1e-13
    assert rel(dW_s, dW_d) < 1e-13 and not np.any(dW_s[~on])
    assert rel(dY_s, dY_d) < 1e-13 and not np.any(dY_s[~on])
    if on.any():
        assert rel(df_s[on], df_d[on]) < 1e-13
    assert not np.any(df_s[~on])


def test_all_ones_and_all_zeros():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax2", 2), n=6, seed=3)
    Y = O.sph_harm(P.L, r)
    E = len(col)
    one, zero = np.ones(E), np.zeros(E)
    assert rel(O.sparse_forward(P, rowptr, col, x, Y, W, one), O.forward(P, rowptr, col, x, Y, W)) < 1e-14
    dx, dW, dY, df = O.sparse_backward(P, rowptr, col, len(x), x, Y, W, one, g)
    rx, rW, rY = O.backward(P, rowptr, col, len(x), x, Y, W, g)
    assert rel(dx, rx) < 1e-14 and rel(dW, rW) < 1e-14 and rel(dY, rY) < 1e-14
    # gate gradient at f = 1: <W, dW> per edge, i.e. <g, the edge's term>
    np.testing.assert_allclose(df, np.sum(W * rW, axis=1), rtol=1e-12, atol=1e-12)
    assert not np.any(O.sparse_forward(P, rowptr, col, x, Y, W, zero))
    for a in O.sparse_backward(P, rowptr, col, len(x), x, Y, W, zero, g):
        assert not np.any(a)


def test_gate_gradient_is_the_derivative_of_the_pairing():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax2_wide", 2), n=6, seed=8)
    Y = O.sph_harm(P.L, r)
    rng = np.random.default_rng(2)
    f = gates(rng, len(col), 0.5)
    S = lambda ff: float(np.sum(g * O.gated_forward(P, rowptr, col, x, Y, W, ff)))
    _, _, _, df_s = O.sparse_backward(P, rowptr, col, len(x), x, Y, W, f, g)
    _, _, _, df_d = O.gated_backward(P, rowptr, col, len(x), x, Y, W, f, g)
    h = 0.25
    for e in range(len(col)):
        fp, fm = f.copy(), f.copy()
        fp[e] += h
        fm[e] -= h
        fd = (S(fp) - S(fm)) / (2 * h)
        assert abs(df_d[e] - fd) <= 1e-10 * max(1.0, abs(fd))
        if f[e] > 0:
            assert abs(df_s[e] - fd) <= 1e-10 * max(1.0, abs(fd))
        else:
            assert df_s[e] == 0.0


def smooth_gate(nu, a=0.4):
    """A C2 gate with an exact flat zero for nu <= a: the quintic smoothstep
    of t = (nu - a) / (1 - a), clamped to [0, 1]."""
    t = np.clip((nu - a) / (1.0 - a), 0.0, 1.0)
    return t ** 3 * (10 - 15 * t + 6 * t ** 2)


def smooth_gate_slope(nu, a=0.4):
    t = np.clip((nu - a) / (1.0 - a), 0.0, 1.0)
    return 30 * t ** 2 * (1 - t) ** 2 / (1.0 - a)


def test_sparse_chain_through_a_flat_gate_is_exact():
    P, rowptr, col, r, x, W, g = problem(shrink("tiny", 2), n=7, seed=4)
    Y = O.sph_harm(P.L, r)
    rng = np.random.default_rng(9)
    nu = rng.uniform(0.0, 1.0, size=len(col))
    nu[np.abs(nu - 0.4) < 0.02] = 0.2  # keep every edge clear of the kink at a
    f = smooth_gate(nu)
    assert np.any(f == 0) and np.any(f > 0)
    _, _, _, df_s = O.sparse_backward(P, rowptr, col, len(x), x, Y, W, f, g)
    dnu = df_s * smooth_gate_slope(nu)
    S = lambda v: float(np.sum(g * O.gated_forward(P, rowptr, col, x, Y, W, smooth_gate(v))))
    h = 1e-6
    for e in range(len(col)):
        vp, vm = nu.copy(), nu.copy()
        vp[e] += h
        vm[e] -= h
        fd = (S(vp) - S(vm)) / (2 * h)
        assert abs(dnu[e] - fd) <= 1e-6 * max(1.0, abs(fd)), (e, nu[e], dnu[e], fd)


def test_planted_threshold_mistake_fails_the_equality_pin():
    P, rowptr, col, r, x, W, g = problem(shrink("lmax2", 2), n=6, seed=1)
    Y = O.sph_harm(P.L, r)
    f = gates(np.random.default_rng(1), len(col), 0.3)
    act = np.nonzero(f >= 0.5)[0]  # the mistake: small non-zero gates dropped
    recv = np.repeat(np.arange(len(rowptr) - 1), np.diff(rowptr))
    rpA = np.concatenate([[0], np.cumsum(np.bincount(recv[act], minlength=len(rowptr) - 1))])
    bad = O.forward(P, rpA, col[act], x, Y[act], f[act, None] * W[act])
    assert rel(bad, O.gated_forward(P, rowptr, col, x, Y, W, f)) > 1e-3
