"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle.

Bar (from the acceptance criteria of the build): rel-L2 <= 1e-5 and
max |err| <= 1e-4 * max |ref| for Y, out, dx, dW and dY; CSR and edge vectors
bit-exact; GPU results bitwise repeatable run to run.  Every workload runs at
its full size (Table 1 Cases 4-6 on the 768-atom cell); the 6144-atom Lmax=3
case is compared on sampled receivers and senders (the oracle computes those
rows exactly from a sub-list of edges).
"""
import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL
from tests._cases import Workload, assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

ALL = ["tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6", "case4", "case5", "case6"]
_plans, _cases = {}, {}


def C():
    from equivariant_mlip_clebsch_b200 import cgtp
    return cgtp


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    return torch.device("cuda:0")


def plan_for(irreps_in, irreps_edge, irreps_out):
    key = (irreps_in, irreps_edge, irreps_out)
    if key not in _plans:
        _plans[key] = C().Plan(irreps_in, irreps_edge, irreps_out, 6)
    return _plans[key]


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


class GpuCase:
    def __init__(self, name, dev):
        w = Workload(name)
        self.w = w
        c = w.cfg
        self.plan = plan_for(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
        rowptr, col, shift, r = C().neighbor_list(w.pos, w.box, c["rc"])
        # the CUDA side's own graph must equal the oracle's bit for bit
        assert np.array_equal(rowptr.astype(np.int64), w.rowptr)
        assert np.array_equal(col, w.col) and np.array_equal(r, w.r32)
        rpt, perm = C().csr_transpose(rowptr, col, w.N)
        self.rowptr, self.col, self.rpt, self.perm = T(rowptr, dev), T(col, dev), T(rpt, dev), T(perm, dev)
        self.r = T(r, dev)
        self.x, self.W, self.g = T(w.x, dev), T(w.W, dev), T(w.g, dev)
        self.Y = self.plan.sph_harm(self.r)
        self.Y_ref = O.sph_harm(w.P.L, w.r32)

    def forward(self):
        return self.plan.forward(self.rowptr, self.col, self.x, self.Y, self.W)

    def backward(self, want=("x", "W", "Y")):
        return self.plan.backward(self.rowptr, self.col, self.rpt, self.perm, self.x, self.Y, self.W,
                                  self.g, want=want)


def case(name, dev):
    if name not in _cases:
        _cases[name] = GpuCase(name, dev)
    return _cases[name]


@pytest.mark.parametrize("name", ALL)
def test_sph_harm(name, dev):
    c = case(name, dev)
    assert_close(c.Y.cpu().numpy(), c.Y_ref, f"{name} Y")


def _receiver_sample(w, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(w.N, size=min(n, w.N), replace=False))


def _sub_csr(w, edge_mask):
    """Receiver CSR over all receivers keeping only the masked edges."""
    recv = np.repeat(np.arange(w.N), np.diff(w.rowptr))
    keep = np.nonzero(edge_mask)[0]
    rp = np.concatenate([[0], np.cumsum(np.bincount(recv[keep], minlength=w.N))]).astype(np.int64)
    return rp, keep


@pytest.mark.parametrize("name", ALL)
def test_forward(name, dev):
    c = case(name, dev)
    w = c.w
    out = c.forward().cpu().numpy()
    c.plan.check_device_error()
    if w.N <= 1024:
        ref = O.forward(w.P, w.rowptr, w.col, w.x, c.Y_ref, w.W)
        assert_close(out, ref, f"{name} out")
    else:
        rows = _receiver_sample(w, 256, 1)
        mask = np.zeros(w.E, bool)
        for i in rows:
            mask[w.rowptr[i]:w.rowptr[i + 1]] = True
        rp, keep = _sub_csr(w, mask)
        ref = O.forward(w.P, rp, w.col[keep], w.x, c.Y_ref[keep], w.W[keep])
        assert_close(out[rows], ref[rows], f"{name} out (256 sampled receivers)")


@pytest.mark.parametrize("name", ALL)
def test_backward(name, dev):
    c = case(name, dev)
    w = c.w
    dx, dW, dY = (t.cpu().numpy() for t in c.backward())
    c.plan.check_device_error()
    if w.N <= 1024:
        rdx, rdW, rdY = O.backward(w.P, w.rowptr, w.col, w.N, w.x, c.Y_ref, w.W, w.g)
        assert_close(dx, rdx, f"{name} dx")
        assert_close(dW, rdW, f"{name} dW")
        assert_close(dY, rdY, f"{name} dY")
    else:
        recv_s = _receiver_sample(w, 128, 2)
        send_s = _receiver_sample(w, 128, 3)
        recv = np.repeat(np.arange(w.N), np.diff(w.rowptr))
        mask = np.isin(recv, recv_s) | np.isin(w.col, send_s)
        rp, keep = _sub_csr(w, mask)
        rdx, rdW, rdY = O.backward(w.P, rp, w.col[keep], w.N, w.x, c.Y_ref[keep], w.W[keep], w.g)
        assert_close(dW[keep], rdW, f"{name} dW (sampled edges)")
        assert_close(dY[keep], rdY, f"{name} dY (sampled edges)")
        assert_close(dx[send_s], rdx[send_s], f"{name} dx (128 sampled senders)")


@pytest.mark.parametrize("name", ["tiny", "lmax2"])
def test_backward_staged_chat(name, dev, monkeypatch):
    """The staged-Chat form of the backward (CGTP_BWD_TFORM=0), kept beside
    the default for comparison, against the oracle."""
    c = case(name, dev)
    w = c.w
    monkeypatch.setenv("CGTP_BWD_TFORM", "0")
    cfg = w.cfg
    plan = C().Plan(cfg["irreps_in"], cfg["irreps_edge"], cfg["irreps_out"], 6)
    assert "backward form=staged_chat" in plan.describe()
    grads = plan.backward(c.rowptr, c.col, c.rpt, c.perm, c.x, c.Y, c.W, c.g)
    plan.check_device_error()
    refs = O.backward(w.P, w.rowptr, w.col, w.N, w.x, c.Y_ref, w.W, w.g)
    for k, a, b in zip("xWY", grads, refs):
        assert_close(a.cpu().numpy(), b, f"{name} d{k} (staged Chat)")


@pytest.mark.parametrize("name", ALL)
def test_force_chain(name, dev):
    """grad_r = dL/dr through the harmonics, and the per-atom forces from it."""
    c = case(name, dev)
    w = c.w
    dYg = np.random.default_rng(7).standard_normal((w.E, w.P.D_e)).astype(np.float32)
    gr = c.plan.sph_harm_backward(c.r, T(dYg, dev))
    ref = O.sph_harm_backward(w.P.L, w.r32, dYg)
    assert_close(gr.cpu().numpy(), ref, f"{name} grad_r")
    # forces on the same FP32 input, then the whole chain
    g32 = ref.astype(np.float32)
    F = C().edge_forces(c.rowptr, c.rpt, c.perm, T(g32, dev)).cpu().numpy()
    assert_close(F, O.edge_forces(w.N, w.rowptr, w.col, g32), f"{name} forces")
    Fc = C().edge_forces(c.rowptr, c.rpt, c.perm, gr).cpu().numpy()
    assert_close(Fc, O.edge_forces(w.N, w.rowptr, w.col, ref), f"{name} forces (chain)")
    assert np.abs(Fc.sum(0)).max() <= 1e-4 * np.abs(Fc).max() * np.sqrt(w.N)  # no net force


@pytest.mark.parametrize("name", ["lmax2", "lmax6"])
def test_bitwise_repeatable(name, dev):
    c = case(name, dev)
    a, b = c.forward().clone(), c.forward().clone()
    assert torch.equal(a, b)
    g1 = [t.clone() for t in c.backward()]
    g2 = [t.clone() for t in c.backward()]
    for p, q in zip(g1, g2):
        assert torch.equal(p, q)


@pytest.mark.parametrize("name", ["lmax2", "lmax3"])
def test_cuda_graph_replay(name, dev):
    """The step (harmonics, forward, backward) captured in a CUDA graph replays
    to the same bits as the launched calls (no allocation or host sync inside
    the calls)."""
    c = case(name, dev)
    w = c.w
    Y = torch.empty_like(c.Y)
    out = torch.empty((w.N, c.plan.d_out), device=dev)
    grads = tuple(torch.empty_like(t) for t in (c.x, c.W, Y))
    ws = torch.empty(max(c.plan.workspace_size(w.N, w.N, w.E), 256), dtype=torch.uint8, device=dev)

    def step():
        c.plan.sph_harm(c.r, Y)
        c.plan.forward(c.rowptr, c.col, c.x, Y, c.W, out=out)
        c.plan.backward(c.rowptr, c.col, c.rpt, c.perm, c.x, Y, c.W, c.g, grads=grads, workspace=ws)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (Y, out) + grads]
    for t in (Y, out) + grads:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    c.plan.check_device_error()
    for a, b in zip(ref, (Y, out) + grads):
        assert torch.equal(a, b)


def test_partial_gradients(dev):
    c = case("lmax2_wide", dev)
    dx, dW, dY = c.backward()
    for want in [("x",), ("W",), ("Y",), ("W", "Y")]:
        got = c.backward(want=want)
        for k, full, part in zip("xWY", (dx, dW, dY), got):
            if k in want:
                assert torch.equal(full, part), (want, k)
            else:
                assert part is None


# ---------------------------------------------------------------- edge cases
RAGGED = [
    ("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o"),                       # partial warps
    ("3x0e+5x1o+2x2e", "1x0e+1x1o+1x2e", None),                        # unaligned rows
    ("96x0e+40x1o", "1x0e+1x1o+1x2e", None),                          # ragged channel blocks
    ("64x0e+64x1o+64x2e+64x3o+64x4e+64x5o+64x6e",
     "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o+1x6e", "lmax6"),                  # several slices
    ("32x0e+17x1o+8x2e+33x3o", "1x0e+1x1o+1x2e+1x3o", None),           # l = 3, partial blocks
]


def _out_irreps(hid, edge):
    P0 = O.enumerate_paths(hid, edge, "+".join(f"1x{l}{p}" for l in range(13) for p in "eo"),
                           check_out=False)
    return "+".join(f"{m}x{l}{'e' if p > 0 else 'o'}" for m, (_, l, p) in
                    zip(P0.out_mul_from_paths, P0.irreps_out) if m > 0)


@pytest.mark.parametrize("spec", RAGGED, ids=["partial_warps", "unaligned", "ragged_blocks", "slices", "l3_partial"])
def test_random_ragged_graphs(spec, dev):
    hid, edge, out = spec
    if out == "lmax6":
        out = WL.CONFIGS["lmax6"]["irreps_out"]
    elif out is None:
        out = _out_irreps(hid, edge)
    check_random_graph(hid, edge, out, dev)


def check_random_graph(hid, edge, out, dev, plan=None):
    """Y, forward and all three gradients on a random ragged graph (37
    receivers, 3 of them without edges, 29 senders, degrees 0-45, one zero
    edge vector) against the oracle."""
    plan = plan or plan_for(hid, edge, out)
    P = O.enumerate_paths(hid, edge, out)
    rng = np.random.default_rng(5)
    n_recv, n_send = 37, 29
    deg = rng.integers(0, 46, size=n_recv)
    deg[[3, 10, 11]] = 0  # receivers without edges
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    E = int(rowptr[-1])
    col = rng.integers(0, n_send, size=E).astype(np.int32)
    r = (rng.standard_normal((E, 3)) * 2).astype(np.float32)
    r[0] = 0.0  # a zero edge vector
    x = rng.standard_normal((n_send, P.D_in)).astype(np.float32)
    W = rng.standard_normal((E, P.U)).astype(np.float32)
    g = rng.standard_normal((n_recv, P.D_out)).astype(np.float32)
    rpt, perm = C().csr_transpose(rowptr.astype(np.int32), col, n_send)
    d = dict(rowptr=T(rowptr.astype(np.int32), dev), col=T(col, dev))
    Y = plan.sph_harm(T(r, dev))
    Y_ref = O.sph_harm(P.L, r)
    assert_close(Y.cpu().numpy(), Y_ref, "Y")
    out_g = plan.forward(d["rowptr"], d["col"], T(x, dev), Y, T(W, dev)).cpu().numpy()
    assert_close(out_g, O.forward(P, rowptr, col, x, Y_ref, W), "out")
    assert np.all(out_g[[3, 10, 11]] == 0)
    grads = plan.backward(d["rowptr"], d["col"], T(rpt, dev), T(perm, dev), T(x, dev), Y, T(W, dev),
                          T(g, dev))
    refs = O.backward(P, rowptr, col, n_send, x, Y_ref, W, g)
    for k, a, b in zip("xWY", grads, refs):
        assert_close(a.cpu().numpy(), b, f"d{k}")
    plan.check_device_error()


@pytest.mark.parametrize("form", ["0", "1"], ids=["scalar_fwd", "packed_fwd"])
@pytest.mark.parametrize("spec", [RAGGED[1], RAGGED[2], RAGGED[4]], ids=["unaligned", "ragged_blocks", "l3_partial"])
def test_forward_forms_on_ragged_graphs(spec, form, dev, monkeypatch):
    """Both forward forms (scalar, and packed FMAs over an m1-major Chat),
    whichever the planner would pick, on ragged graphs and channel blocks."""
    hid, edge, out = spec
    out = out or _out_irreps(hid, edge)
    monkeypatch.setenv("CGTP_FWD_PACKED", form)
    plan = C().Plan(hid, edge, out, 6)
    assert ("forward form=packed" in plan.describe()) == (form == "1")
    check_random_graph(hid, edge, out, dev, plan)


def test_empty_graph(dev):
    plan = plan_for("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o")
    rowptr = torch.zeros(6, dtype=torch.int32, device=dev)
    col = torch.zeros(0, dtype=torch.int32, device=dev)
    x = torch.randn(4, plan.d_in, device=dev)
    Y = torch.zeros(0, plan.d_edge, device=dev)
    W = torch.zeros(0, plan.n_weights, device=dev)
    out = plan.forward(rowptr, col, x, Y, W)
    assert out.shape == (5, plan.d_out) and torch.count_nonzero(out) == 0
    rpt = torch.zeros(5, dtype=torch.int32, device=dev)
    g = torch.randn(5, plan.d_out, device=dev)
    dx, dW, dY = plan.backward(rowptr, col, rpt, col, x, Y, W, g)
    assert torch.count_nonzero(dx) == 0 and dW.numel() == 0 and dY.numel() == 0


def test_argument_errors(dev):
    plan = plan_for("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o")
    rowptr = torch.zeros(3, dtype=torch.int32, device=dev)
    x = torch.randn(2, plan.d_in, device=dev)
    buf = torch.zeros(2 * plan.d_out + 1, device=dev)
    with pytest.raises(C().CgtpError) as e:  # misaligned output
        plan.forward(rowptr, rowptr[:0], x, x[:0], x[:0], out=buf[1:].view(2, plan.d_out))
    assert e.value.status == 2
    ws = torch.zeros(16, dtype=torch.uint8, device=dev)
    rp = torch.tensor([0, 1, 1], dtype=torch.int32, device=dev)
    col = torch.zeros(1, dtype=torch.int32, device=dev)
    with pytest.raises(C().CgtpError) as e:  # workspace too small for grad_x
        plan.backward(rp, col, torch.tensor([0, 1, 1], dtype=torch.int32, device=dev), col, x,
                      torch.zeros(1, plan.d_edge, device=dev), torch.zeros(1, plan.n_weights, device=dev),
                      torch.zeros(2, plan.d_out, device=dev), workspace=ws)
    assert e.value.status == 12
