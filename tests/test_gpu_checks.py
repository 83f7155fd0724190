"""Device checks of the graph, and the kernels' wind-down after a wait
expires (GPU, tiny workload only).

Graph checks (cgtp_plan_set_checks): a col entry past n_send, a decreasing
rowptr and a perm_T entry that lists another sender's edge each make the
call return CGTP_ERR_INVALID_CSR before any kernel reads through the graph.
Every bad case keeps each index inside the buffers it would address (x has
rows up to the largest col written, rowptr stays within [0, E], perm_T
values stay within [0, E)), so that a check that failed to fire would still
read in bounds.  The next valid call on the same plan matches the oracle.

Wind-down: a plan compiled with a pipeline-wait limit of a few polls
(CGTP_SPIN_LIMIT at plan creation) makes waits expire; the kernels record
CGTP_ERR_TIMEOUT in the plan's error word (or nothing, if no wait had to
wait) and return; the TMA warp still drains its own copies before the CTA
exits.  A normal plan's next call then matches the oracle.
"""
import numpy as np
import pytest

import oracle as O
from tests._cases import Workload, assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def C():
    from equivariant_mlip_clebsch_b200 import cgtp
    return cgtp


@pytest.fixture(scope="module")
def tiny():
    dev = torch.device("cuda:0")
    w = Workload("tiny")
    c = w.cfg
    plan = C().Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    rowptr, col, shift, r = C().neighbor_list(w.pos, w.box, c["rc"])
    rpt, perm = C().csr_transpose(rowptr, col, w.N)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    d = dict(rowptr=rowptr, col=col, rpt=rpt, perm=perm, T=T, dev=dev)
    d["Y"] = plan.sph_harm(T(r))
    Yr = O.sph_harm(w.P.L, w.r32)
    d["ref_out"] = O.forward(w.P, w.rowptr, w.col, w.x, Yr, w.W)
    d["ref_bwd"] = O.backward(w.P, w.rowptr, w.col, w.N, w.x, Yr, w.W, w.g)
    return w, plan, d


def _valid_calls(w, plan, d):
    T = d["T"]
    out = plan.forward(T(d["rowptr"]), T(d["col"]), T(w.x), d["Y"], T(w.W))
    grads = plan.backward(T(d["rowptr"]), T(d["col"]), T(d["rpt"]), T(d["perm"]), T(w.x), d["Y"], T(w.W), T(w.g))
    torch.cuda.synchronize()
    plan.check_device_error()
    assert_close(out.cpu().numpy(), d["ref_out"], "out")
    for k, a, b in zip("xWY", grads, d["ref_bwd"]):
        assert_close(a.cpu().numpy(), b, f"d{k}")


def test_graph_checks_refuse_bad_graphs(tiny):
    w, plan, d = tiny
    T = d["T"]
    plan.set_checks(True)
    try:
        _valid_calls(w, plan, d)  # a valid graph passes the checks
        # 1. col entries at n_send and beyond; x holds rows for all of them
        col = d["col"].copy()
        col[5], col[100] = w.N, w.N + 3
        x_big = np.zeros((w.N + 4, plan.d_in), np.float32)
        x_big[:w.N] = w.x
        import ctypes
        rp_t, col_t, x_t, W_t = T(d["rowptr"]), T(col), T(x_big), T(w.W)
        out = torch.empty((w.N, plan.d_out), device=d["dev"])
        P = lambda t: ctypes.c_void_p(t.data_ptr())
        # n_send = N (the graph's senders) while x holds N + 4 rows
        st = C()._lib.cgtp_forward(plan._h, w.N, w.N, w.E, P(rp_t), P(col_t), P(x_t), P(d["Y"]), P(W_t), P(out),
                                   C()._stream())
        assert st == 7 and "col" in C()._lib.cgtp_last_error().decode()
        # 2. a decreasing rowptr, every entry still inside [0, E]
        rp = d["rowptr"].copy()
        rp[10], rp[11] = rp[11], rp[10]
        assert rp[10] > rp[11]
        with pytest.raises(C().CgtpError) as e:
            plan.backward(T(rp), T(d["col"]), T(d["rpt"]), T(d["perm"]), T(w.x), d["Y"], T(w.W), T(w.g))
        assert e.value.status == 7 and "rowptr decreases" in str(e.value)
        # 3. perm_T with two entries of different senders exchanged (values in [0, E))
        perm = d["perm"].copy()
        a, b = d["rpt"][3], d["rpt"][40]
        perm[a], perm[b] = perm[b], perm[a]
        with pytest.raises(C().CgtpError) as e:
            plan.backward(T(d["rowptr"]), T(d["col"]), T(d["rpt"]), T(perm), T(w.x), d["Y"], T(w.W), T(w.g))
        assert e.value.status == 7 and "perm_T" in str(e.value)
        # without grad_x the sender lists are not read, and not checked
        plan.backward(T(d["rowptr"]), T(d["col"]), T(d["rpt"]), T(perm), T(w.x), d["Y"], T(w.W), T(w.g),
                      want=("W", "Y"))
        # 4. the next valid calls still match the oracle
        _valid_calls(w, plan, d)
    finally:
        plan.set_checks(False)


def test_validate_graph(tiny):
    """cgtp_validate_graph runs the same checks once, whatever the plan's
    flags: a valid graph passes, a bad col, rowptr or perm_T is named."""
    w, plan, d = tiny
    T = d["T"]
    plan.validate_graph(T(d["rowptr"]), T(d["col"]), w.N)
    plan.validate_graph(T(d["rowptr"]), T(d["col"]), w.N, T(d["rpt"]), T(d["perm"]))
    col = d["col"].copy()
    col[7] = w.N
    with pytest.raises(C().CgtpError) as e:
        plan.validate_graph(T(d["rowptr"]), T(col), w.N)
    assert e.value.status == 7 and "col" in str(e.value)
    rp = d["rowptr"].copy()
    rp[10], rp[11] = rp[11], rp[10]
    with pytest.raises(C().CgtpError) as e:
        plan.validate_graph(T(rp), T(d["col"]), w.N)
    assert e.value.status == 7 and "rowptr decreases" in str(e.value)
    perm = d["perm"].copy()
    a, b = d["rpt"][3], d["rpt"][40]
    perm[a], perm[b] = perm[b], perm[a]
    with pytest.raises(C().CgtpError) as e:
        plan.validate_graph(T(d["rowptr"]), T(d["col"]), w.N, T(d["rpt"]), T(perm))
    assert e.value.status == 7 and "perm_T" in str(e.value)
    _valid_calls(w, plan, d)  # the plan's own calls are unaffected


def test_checks_flags_are_validated(tiny):
    w, plan, d = tiny
    with pytest.raises(C().CgtpError) as e:
        C()._check(C()._lib.cgtp_plan_set_checks(plan._h, 6))
    assert e.value.status == 6


@pytest.mark.parametrize("limit", [1, 16])
def test_expired_waits_wind_down(tiny, monkeypatch, limit):
    w, plan, d = tiny
    T = d["T"]
    monkeypatch.setenv("CGTP_SPIN_LIMIT", str(limit))
    c = w.cfg
    short = C().Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    monkeypatch.delenv("CGTP_SPIN_LIMIT")
    codes = []
    for _ in range(3):
        short.forward(T(d["rowptr"]), T(d["col"]), T(w.x), d["Y"], T(w.W))
        short.backward(T(d["rowptr"]), T(d["col"]), T(d["rpt"]), T(d["perm"]), T(w.x), d["Y"], T(w.W), T(w.g))
        torch.cuda.synchronize()  # the context is still usable
        try:
            short.check_device_error()
            codes.append(0)
        except C().CgtpError as e:
            assert e.value.status == 10  # CGTP_ERR_TIMEOUT
            codes.append(10)
    short.close()
    # the ordinary plan is unaffected
    _valid_calls(w, plan, d)
