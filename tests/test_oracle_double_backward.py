"""Pins of the oracle's double backward (the gradients of a functional of
the backward's outputs: the second-order pass that force and Hessian
training run through the CGTP convolution; LunaTP Table 11 lists its outputs
h_x and h_y beside the forward's and backward's).

S(g, x, Y, W) = <h_x, dx> + <h_W, dW> + <h_Y, dY>, with (dx, dW, dY) the
oracle's backward, is linear in each of g, x, Y and W separately, so a
central difference along any direction equals the directional derivative up
to rounding.  The oracle's double backward (written as forwards and
backwards with one argument replaced by its cotangent) must match those
differences for every subset of cotangents; with a term dropped it does not.
"""
import itertools

import numpy as np
import pytest

import oracle as O
from tests.test_oracle_conv import problem, shrink


def _setup(name="lmax3", n=6, seed=3):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 2), n=n, seed=seed)
    Y = O.sph_harm(P.L, r)
    rng = np.random.default_rng(seed + 100)
    h = dict(h_x=rng.standard_normal(x.shape), h_W=rng.standard_normal(W.shape),
             h_Y=rng.standard_normal(Y.shape))
    return P, rowptr, col, n, x, Y, W, g, h, rng


def _S(P, rowptr, col, n, x, Y, W, g, h):
    dx, dW, dY = O.backward(P, rowptr, col, n, x, Y, W, g)
    s = 0.0
    for key, d in (("h_x", dx), ("h_W", dW), ("h_Y", dY)):
        if h.get(key) is not None:
            s += float((h[key] * d).sum())
    return s


@pytest.mark.parametrize("keys", [k for m in range(1, 4) for k in itertools.combinations(("h_x", "h_W", "h_Y"), m)])
def test_directional_differences(keys):
    P, rowptr, col, n, x, Y, W, g, hall, rng = _setup()
    h = {k: (hall[k] if k in keys else None) for k in hall}
    gg, gx, gW, gY = O.double_backward(P, rowptr, col, n, x, Y, W, g, **h)
    args = dict(x=x, Y=Y, W=W, g=g)
    for name, grad in (("g", gg), ("x", gx), ("W", gW), ("Y", gY)):
        d = rng.standard_normal(args[name].shape)
        plus, minus = dict(args), dict(args)
        plus[name] = args[name] + d
        minus[name] = args[name] - d
        fd = (_S(P, rowptr, col, n, h=h, **plus) - _S(P, rowptr, col, n, h=h, **minus)) / 2.0
        assert fd == pytest.approx(float((grad * d).sum()), rel=1e-10, abs=1e-9), (keys, name)


def test_absent_cotangents_give_zero_terms():
    """With only h_Y, S = <g, fwd(x, h_Y, W)> does not depend on Y."""
    P, rowptr, col, n, x, Y, W, g, h, _ = _setup("lmax2")
    gg, gx, gW, gY = O.double_backward(P, rowptr, col, n, x, Y, W, g, h_Y=h["h_Y"])
    assert np.all(gY == 0.0)
    assert np.allclose(gg, O.forward(P, rowptr, col, x, h["h_Y"], W), atol=1e-12)


def test_pin_catches_a_dropped_term():
    P, rowptr, col, n, x, Y, W, g, h, rng = _setup()
    gg, gx, gW, gY = O.double_backward(P, rowptr, col, n, x, Y, W, g, **h)
    # planted mistake: the Y gradient without the h_W term
    _, _, _, gY_wrong = O.double_backward(P, rowptr, col, n, x, Y, W, g, h_x=h["h_x"], h_Y=h["h_Y"])
    d = rng.standard_normal(Y.shape)
    fd = (_S(P, rowptr, col, n, x, Y + d, W, g, h) - _S(P, rowptr, col, n, x, Y - d, W, g, h)) / 2.0
    assert fd == pytest.approx(float((gY * d).sum()), rel=1e-10, abs=1e-9)
    assert abs(fd - float((gY_wrong * d).sum())) > 1e-3 * abs(fd)
