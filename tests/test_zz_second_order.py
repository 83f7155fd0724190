"""GPU parity of the double backward (cgtp_double_backward) against the
oracle's, which tests/test_oracle_double_backward.py pins to directional
differences of S = <h_x, dx> + <h_W, dW> + <h_Y, dY>.  Random ragged graphs
with several subsets of cotangents, and two workloads at full size; both
sides take the same FP32 inputs.  Same bar as the other parity tests.
Named to be collected after them.
"""
import numpy as np
import pytest

import oracle as O
from tests._cases import assert_close
from tests.test_gpu_parity import T, _out_irreps, case, plan_for

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    return torch.device("cuda:0")


def _compare(plan, P, d, host, h, dev):
    """Run the GPU double backward on device arrays d and the oracle on the
    same host arrays; compare the four gradients."""
    hd = {k: (None if v is None else T(v, dev)) for k, v in h.items()}
    got = plan.double_backward(d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], d["Y"], d["W"], d["g"], **hd)
    ref = O.double_backward(P, host["rowptr"], host["col"], host["n_send"], host["x"], host["Y"], host["W"],
                            host["g"], **h)
    for name, a, b in zip(("d grad_out", "dx", "dW", "dY"), got, ref):
        assert_close(a.cpu().numpy(), b, name)
    plan.check_device_error()
    return got


@pytest.mark.parametrize("keys", [("h_x", "h_W", "h_Y"), ("h_x",), ("h_W",), ("h_Y",), ("h_W", "h_Y")])
def test_double_backward_random_graph(keys, dev):
    hid, edge = "96x0e+40x1o", "1x0e+1x1o+1x2e"
    out = _out_irreps(hid, edge)
    _random_graph_case(plan_for(hid, edge, out), hid, edge, out, keys, dev)


@pytest.mark.parametrize("fwd", ["tangent", "sum"])
@pytest.mark.parametrize("hid,edge", [("96x0e+40x1o", "1x0e+1x1o+1x2e"),
                                      ("32x0e+17x1o+8x2e+33x3o", "1x0e+1x1o+1x2e+1x3o")],
                         ids=["l1", "l3_partial"])
def test_double_backward_forward_paths(hid, edge, fwd, dev, monkeypatch):
    """Both ways of forming d grad_out: the tangent forward, and one plain
    plus two accumulating forwards (the planner's choice for plans with packed
    forward roles)."""
    out = _out_irreps(hid, edge)
    monkeypatch.setenv("CGTP_DBWD_FWD", fwd)
    from equivariant_mlip_clebsch_b200 import cgtp as C
    plan = C.Plan(hid, edge, out, 6)
    assert plan.prepare_double_backward()
    assert ("cgtp_fwd_acc" in plan.describe()) == (fwd == "sum")
    _random_graph_case(plan, hid, edge, out, ("h_x", "h_W", "h_Y"), dev)


def test_double_backward_first_call_chooses(dev, monkeypatch):
    """With both ways of forming d grad_out built, the first call times them
    and keeps the faster; that call and the next give the same bits."""
    monkeypatch.delenv("CGTP_DBWD_FWD", raising=False)  # the choice is the plan's
    hid, edge = "32x0e+17x1o+8x2e+33x3o", "1x0e+1x1o+1x2e+1x3o"
    out = _out_irreps(hid, edge)
    from equivariant_mlip_clebsch_b200 import cgtp as C
    plan = C.Plan(hid, edge, out, 6)
    assert plan.prepare_double_backward()
    assert "double backward forward=undecided" in plan.describe()
    first = _random_graph_case(plan, hid, edge, out, ("h_x", "h_W", "h_Y"), dev)
    desc = plan.describe()
    assert "double backward forward=tangent" in desc or "double backward forward=sum" in desc
    second = _random_graph_case(plan, hid, edge, out, ("h_x", "h_W", "h_Y"), dev)
    for a, b in zip(first, second):
        assert torch.equal(a, b)


def _random_graph_case(plan, hid, edge, out, keys, dev):
    P = O.enumerate_paths(hid, edge, out)
    rng = np.random.default_rng(11)
    n_recv, n_send = 37, 29
    deg = rng.integers(0, 46, size=n_recv)
    deg[[3, 10, 11]] = 0
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    E = int(rowptr[-1])
    col = rng.integers(0, n_send, size=E).astype(np.int32)
    r = (rng.standard_normal((E, 3)) * 2).astype(np.float32)
    Y = O.sph_harm(P.L, r).astype(np.float32)
    f32 = lambda *s: rng.standard_normal(s).astype(np.float32)
    host = dict(rowptr=rowptr, col=col, n_send=n_send, x=f32(n_send, P.D_in), Y=Y, W=f32(E, P.U),
                g=f32(n_recv, P.D_out))
    h = dict(h_x=f32(n_send, P.D_in) if "h_x" in keys else None, h_W=f32(E, P.U) if "h_W" in keys else None,
             h_Y=f32(E, P.D_e) if "h_Y" in keys else None)
    from equivariant_mlip_clebsch_b200 import cgtp as C
    rpt, perm = C.csr_transpose(rowptr.astype(np.int32), col, n_send)
    d = dict(rowptr=T(rowptr.astype(np.int32), dev), col=T(col, dev), rpt=T(rpt, dev), perm=T(perm, dev),
             x=T(host["x"], dev), Y=T(Y, dev), W=T(host["W"], dev), g=T(host["g"], dev))
    return _compare(plan, P, d, host, h, dev)


@pytest.mark.parametrize("name", ["tiny", "lmax2"])
def test_double_backward_workload(name, dev):
    c = case(name, dev)
    w = c.w
    rng = np.random.default_rng(12)
    Y = c.Y.cpu().numpy()
    host = dict(rowptr=w.rowptr, col=w.col, n_send=w.N, x=w.x, Y=Y, W=w.W, g=w.g)
    h = dict(h_x=rng.standard_normal(w.x.shape).astype(np.float32),
             h_W=rng.standard_normal(w.W.shape).astype(np.float32),
             h_Y=rng.standard_normal(Y.shape).astype(np.float32))
    d = dict(rowptr=c.rowptr, col=c.col, rpt=c.rpt, perm=c.perm, x=c.x, Y=c.Y, W=c.W, g=c.g)
    _compare(c.plan, w.P, d, host, h, dev)
