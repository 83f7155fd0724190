"""GPU parity of the BranchIP sparse evaluation (through the C ABI).

The sparse forward and backward (zero-gated edges skipped, per-edge outputs
zero-padded to the full edge set) against the oracle's sparse evaluation,
which its CPU tests pin to the dense gated evaluation (BranchIP page, section
"BranchIP": the sparse path reproduces the dense one).  Workloads at full
size, 25 / 50 / 75 % active edges, all edges active (then bitwise equal to
the plain convolution: a gate of one changes no value), none active, and
random ragged graphs; skipped edges' rows are checked to be exactly zero.
"""
import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL
from tests._cases import Workload, assert_close
from tests.test_oracle_conv import problem, shrink

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

_plans = {}


def C():
    from equivariant_mlip_clebsch_b200 import cgtp
    return cgtp


def plan_for(a, b, c):
    if (a, b, c) not in _plans:
        _plans[(a, b, c)] = C().Plan(a, b, c, 6)
    return _plans[(a, b, c)]


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available()
    return torch.device("cuda:0")


def _run_and_check(plan, P, rowptr, col, x, Yr, Ygpu, W, g, gate, n_send, dev, what):
    rpt, perm = C().csr_transpose(rowptr.astype(np.int32), col.astype(np.int32), n_send)
    d = dict(rowptr=T(rowptr.astype(np.int32), dev), col=T(col.astype(np.int32), dev), rpt=T(rpt, dev),
             perm=T(perm, dev), x=T(x, dev), W=T(W, dev), g=T(g, dev), f=T(gate, dev))
    out = plan.sparse_forward(d["rowptr"], d["col"], d["x"], Ygpu, d["W"], d["f"])
    dx, dW, dY, df = plan.sparse_backward(d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], Ygpu, d["W"],
                                          d["f"], d["g"])
    torch.cuda.synchronize()
    plan.check_device_error()
    ref_out = O.sparse_forward(P, rowptr, col, x, Yr, W, gate.astype(np.float64))
    rdx, rdW, rdY, rdf = O.sparse_backward(P, rowptr, col, n_send, x, Yr, W, gate.astype(np.float64), g)
    off = gate <= 0
    got = [t.cpu().numpy() for t in (out, dx, dW, dY, df)]
    for nm, a, b in zip(["out", "dx", "dW", "dY", "dgate"], got, [ref_out, rdx, rdW, rdY, rdf]):
        if np.any(b):
            assert_close(a, b, f"{what} sparse {nm}")
        else:
            assert not np.any(a), f"{what} sparse {nm}: expected zeros"
    for nm, a in zip(["dW", "dY", "dgate"], got[2:]):
        assert not np.any(a[off]), f"{what}: {nm} of skipped edges not zero"
    return d, got


@pytest.mark.parametrize("name", ["tiny", "lmax2", "lmax2_wide"])
@pytest.mark.parametrize("frac", [0.25, 0.5, 0.75])
def test_sparse_matches_the_oracle(name, frac, dev):
    w = Workload(name)
    c = w.cfg
    plan = plan_for(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    gate = WL.draw_gate(w.E, frac)
    Yr = O.sph_harm(w.P.L, w.r32)
    Ygpu = plan.sph_harm(T(w.r32, dev))
    _run_and_check(plan, w.P, w.rowptr, w.col, w.x, Yr, Ygpu, w.W, w.g, gate, w.N, dev, f"{name} {frac}")


def test_all_active_is_the_plain_convolution_bit_for_bit(dev):
    w = Workload("lmax2")
    c = w.cfg
    plan = plan_for(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    Ygpu = plan.sph_harm(T(w.r32, dev))
    Yr = O.sph_harm(w.P.L, w.r32)
    gate = np.ones(w.E, dtype=np.float32)
    d, got = _run_and_check(plan, w.P, w.rowptr, w.col, w.x, Yr, Ygpu, w.W, w.g, gate, w.N, dev, "lmax2 all")
    out = plan.forward(d["rowptr"], d["col"], d["x"], Ygpu, d["W"])
    dx, dW, dY = plan.backward(d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], Ygpu, d["W"], d["g"])
    torch.cuda.synchronize()
    for nm, a, b in zip(["out", "dx", "dW", "dY"], got[:4], (out, dx, dW, dY)):
        assert np.array_equal(a, b.cpu().numpy()), f"all-active sparse {nm} differs from the plain path"


def test_none_active_gives_zeros(dev):
    w = Workload("tiny")
    c = w.cfg
    plan = plan_for(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    Ygpu = plan.sph_harm(T(w.r32, dev))
    Yr = O.sph_harm(w.P.L, w.r32)
    gate = np.zeros(w.E, dtype=np.float32)
    _, got = _run_and_check(plan, w.P, w.rowptr, w.col, w.x, Yr, Ygpu, w.W, w.g, gate, w.N, dev, "tiny none")
    for a in got:
        assert not np.any(a)


@pytest.mark.parametrize("name,seed", [("lmax2", 1), ("lmax2_wide", 2), ("lmax3", 3), ("tiny", 4)])
def test_sparse_on_random_ragged_graphs(name, seed, dev):
    P, rowptr, col, r, x, W, g = problem(shrink(name, 33), n=57, seed=seed, max_deg=11)
    hid, edge, out_ir = shrink(name, 33)
    plan = plan_for(hid, edge, out_ir)
    r32 = r.astype(np.float32)
    Yr = O.sph_harm(P.L, r32)
    Ygpu = plan.sph_harm(T(r32, dev))
    x, W, g = x.astype(np.float32), W.astype(np.float32), g.astype(np.float32)
    gate = WL.draw_gate(len(col), 0.4, seed)
    _run_and_check(plan, P, rowptr, col, x, Yr, Ygpu, W, g, gate, len(x), dev, f"ragged {name}")
