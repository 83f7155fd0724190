"""The backward entry point that allocates nothing.

cgtp_backward_static_scratch serves callers that cannot allocate device
memory when they run the backward (an engine that sizes all of its memory at
start-up, a runtime without a device allocator): its scratch is a fixed array
in the library's device code instead of a caller workspace.  These checks call
it through the C ABI twice in a row and compare each result with the ordinary
cgtp_backward on the same inputs, with the tolerance of the other parity
tests, and check that sizes beyond the fixed array are refused.  The file is
named to be collected last.
"""
import numpy as np
import pytest

from equivariant_mlip_clebsch_b200 import workloads as WL
from tests._cases import assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _setup(name, dev):
    from equivariant_mlip_clebsch_b200 import cgtp as C
    c = WL.CONFIGS[name]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    pos, box = WL.si_diamond(c["cells"], c["sigma"], 0)
    rowptr, col, shift, r = C.neighbor_list(pos, box, c["rc"])
    N, E = len(pos), len(col)
    rpt, perm = C.csr_transpose(rowptr, col, N)
    muls = [int(t.split("x")[0]) for t in c["irreps_out"].split("+")]
    std = WL.column_std(muls, plan.out_fan_in())
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    d = dict(rowptr=T(rowptr), col=T(col), rpt=T(rpt), perm=T(perm), x=T(WL.draw_x(N, plan.d_in)),
             W=T(WL.draw_W(E, plan.n_weights, std)), g=T(WL.draw_g(N, plan.d_out)))
    d["Y"] = plan.sph_harm(T(r))
    return C, plan, d, N, E


@pytest.mark.parametrize("name", ["tiny", "lmax2"])
def test_static_scratch_matches_workspace_backward(name):
    dev = torch.device("cuda:0")
    C, plan, d, N, E = _setup(name, dev)
    args = (d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], d["Y"], d["W"], d["g"])
    ref = [t.clone() for t in plan.backward(*args)]
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the fixed scratch
        grads = (torch.full_like(ref[0], np.nan), torch.full_like(ref[1], np.nan),
                 torch.full_like(ref[2], np.nan))
        got = plan.backward_static_scratch(*args, grads=grads)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in got])
    plan.check_device_error()
    for call in outs:
        for k, a, b in zip("xWY", call, ref):
            assert_close(a.cpu().numpy(), b.cpu().numpy(), f"{name} d{k} (static scratch)")


def test_static_scratch_rejects_sizes_beyond_the_array():
    dev = torch.device("cuda:0")
    C, plan, d, N, E = _setup("lmax2_wide", dev)
    assert plan.workspace_size(N, N, E) > C.STATIC_SCRATCH_BYTES
    with pytest.raises(C.CgtpError) as e:
        plan.backward_static_scratch(d["rowptr"], d["col"], d["rpt"], d["perm"], d["x"], d["Y"],
                                     d["W"], d["g"])
    assert e.value.status == 12
