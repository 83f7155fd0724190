"""The backward entry point that allocates nothing.

cgtp_backward_static_scratch serves callers that cannot allocate device
memory when they run the backward: an engine that sizes all of its device
memory once at start-up and forbids allocation afterwards, or a runtime that
owns no device allocator and must not pull one in.  Its scratch is a fixed
array in the library's device code instead of a caller workspace.

These checks call it through the C ABI and compare every result with the FP64
oracle (the tolerance of the other parity tests), two calls in a row (the
array keeps the first call's contents), for each subset of gradients (each
uses a different part of the array), on a second stream ordered by an event,
and check that a call needing more scratch than the array holds is refused
while a grad_W-only call on the same large graph, which needs none, runs.
The file is named to be collected after every other test.
"""
import numpy as np
import pytest

import oracle as O
from tests._cases import Workload, assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

_setups = {}


def _setup(name, dev):
    if name in _setups:
        return _setups[name]
    from equivariant_mlip_clebsch_b200 import cgtp as C
    w = Workload(name)
    c = w.cfg
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    rowptr, col, shift, r = C.neighbor_list(w.pos, w.box, c["rc"])
    assert np.array_equal(rowptr.astype(np.int64), w.rowptr) and np.array_equal(col, w.col)
    rpt, perm = C.csr_transpose(rowptr, col, w.N)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    d = dict(rowptr=T(rowptr), col=T(col), rpt=T(rpt), perm=T(perm), x=T(w.x), W=T(w.W), g=T(w.g))
    d["Y"] = plan.sph_harm(T(r))
    ref = None
    if w.N <= 1024:
        Yr = O.sph_harm(w.P.L, w.r32)
        ref = O.backward(w.P, w.rowptr, w.col, w.N, w.x, Yr, w.W, w.g)
    _setups[name] = (C, plan, d, w, ref)
    return _setups[name]


def _args(d):
    return (d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], d["Y"], d["W"], d["g"])


@pytest.mark.parametrize("name,want", [
    ("tiny", ("x", "W", "Y")), ("tiny", ("x",)), ("tiny", ("W",)), ("tiny", ("Y",)), ("tiny", ("x", "Y")),
    ("lmax2", ("x", "W", "Y")), ("lmax2", ("Y",))])
def test_static_scratch_matches_the_oracle(name, want):
    dev = torch.device("cuda:0")
    C, plan, d, w, ref = _setup(name, dev)
    shapes = ((w.N, plan.d_in), (w.E, plan.n_weights), (w.E, plan.d_edge))
    for call in range(2):  # two calls in a row share (and reuse) the fixed array
        grads = tuple(torch.full(s, float("nan"), device=dev) if k in want else None
                      for k, s in zip("xWY", shapes))
        got = plan.backward_static_scratch(*_args(d), grads=grads)
        torch.cuda.synchronize()
        plan.check_device_error()
        for k, a, b in zip("xWY", got, ref):
            if k in want:
                assert_close(a.cpu().numpy(), b, f"{name} d{k} want={want} call {call} (static scratch)")
            else:
                assert a is None


def test_static_scratch_on_a_second_stream():
    dev = torch.device("cuda:0")
    C, plan, d, w, ref = _setup("tiny", dev)
    s = torch.cuda.Stream(dev)
    ready = torch.cuda.Event()
    ready.record(torch.cuda.current_stream())
    s.wait_event(ready)
    got = plan.backward_static_scratch(*_args(d), stream=s)
    done = torch.cuda.Event()
    done.record(s)
    torch.cuda.current_stream().wait_event(done)
    torch.cuda.synchronize()
    plan.check_device_error()
    for k, a, b in zip("xWY", got, ref):
        assert_close(a.cpu().numpy(), b, f"tiny d{k} (static scratch, second stream)")


def test_static_scratch_refuses_what_does_not_fit_and_runs_what_needs_none():
    dev = torch.device("cuda:0")
    C, plan, d, w, ref = _setup("lmax2_wide", dev)
    assert plan.workspace_size(w.N, w.N, w.E) > C.STATIC_SCRATCH_BYTES
    with pytest.raises(C.CgtpError) as e:
        plan.backward_static_scratch(*_args(d))
    assert e.value.status == 12
    # grad_W alone needs no scratch: it runs on the same graph and matches
    # the workspace backward's grad_W (checked against the oracle elsewhere)
    _, dW, _ = plan.backward_static_scratch(*_args(d), want=("W",))
    _, dW_ref, _ = plan.backward(*_args(d), want=("W",))
    torch.cuda.synchronize()
    plan.check_device_error()
    assert torch.equal(dW, dW_ref)
