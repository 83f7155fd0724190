"""GPU parity of the strain derivative (virial), cgtp_edge_virial.

V[a,b] = sum_e grad_r[e,a] r[e,b] against the FP64 oracle (pinned in
tests/test_oracle_forces.py to finite differences of a strained energy):
  * on random FP32 edges, with every tail length E % 4 and E = 0 (zeros);
  * at the end of the force chain on the workloads (grad_r from the
    harmonics' backward), where the trace also vanishes because the
    harmonics depend on the direction alone;
  * bitwise repeatable (the summation order depends on E only).
Same bar as the other parity tests.  Named to be collected after them.
"""
import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL
from tests._cases import assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    return torch.device("cuda:0")


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


@pytest.mark.parametrize("E", [0, 1, 2, 3, 4, 5, 4099, 16387, 172050])
def test_virial_random_edges(E, dev):
    from equivariant_mlip_clebsch_b200 import cgtp as C
    rng = np.random.default_rng(100 + E)
    r = (2.0 * rng.standard_normal((E, 3))).astype(np.float32)
    G = rng.standard_normal((E, 3)).astype(np.float32)
    V = C.edge_virial(T(r, dev), T(G, dev))
    assert V.shape == (3, 3)
    got = V.cpu().numpy()
    if E == 0:
        assert np.all(got == 0.0)
    else:
        assert_close(got, O.edge_virial(r, G), f"virial E={E}")
    again = C.edge_virial(T(r, dev), T(G, dev)).cpu().numpy()
    assert np.array_equal(got, again)


@pytest.mark.parametrize("name", ["tiny", "lmax2", "lmax6"])
def test_virial_force_chain(name, dev):
    from equivariant_mlip_clebsch_b200 import cgtp as C
    c = WL.CONFIGS[name]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    L = int(round(np.sqrt(plan.d_edge))) - 1
    pos, box = WL.si_diamond(c["cells"], c["sigma"], 0)
    _, col, _, r = C.neighbor_list(pos, box, c["rc"])
    dY = np.random.default_rng(17).standard_normal((len(col), plan.d_edge)).astype(np.float32)
    rt = T(r, dev)
    gr = plan.sph_harm_backward(rt, T(dY, dev))
    V = C.edge_virial(rt, gr).cpu().numpy()
    ref = O.edge_virial(r, O.sph_harm_backward(L, r, dY))
    assert_close(V, ref, f"{name} virial (chain)")
    assert abs(np.trace(V)) <= 1e-4 * np.abs(V).max()
    plan.check_device_error()
