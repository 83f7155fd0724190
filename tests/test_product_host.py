"""Host-side checks of libcgtp that need no GPU.

  * the library loads and exports every entry point include/cgtp.h declares;
  * its real CG blocks (ladder-operator construction) equal the oracle's
    (Racah closed form) -- two independent routes to the same table;
  * its cell-list neighbour list equals the oracle's brute force bit for bit,
    edge vectors included;
  * the CSR transpose and the host argument checks;
  * every workload's plan builds and its kernels compile for sm_100a (the
    compile-only mode skips all device work), with the oracle's path table.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from equivariant_mlip_clebsch_b200 import workloads as WL
from equivariant_mlip_clebsch_b200 import cgtp as C

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "cgtp.h")


def test_every_declared_symbol_is_exported():
    decl = set(re.findall(r"^\s*(?:const char\*|cgtp_status)\s+(cgtp_\w+)\s*\(", open(HEADER).read(), re.M))
    assert len(decl) >= 15
    for name in decl:
        assert hasattr(C._lib, name), name
    assert decl == set(C.EXPORTS)


def test_real_cg_matches_oracle_all_triples():
    for l1 in range(7):
        for l2 in range(7):
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                a = C.real_cg(l1, l2, l3)
                b = O.real_cg(l1, l2, l3)
                assert np.allclose(a, b, atol=1e-12), (l1, l2, l3)
                assert np.array_equal(a == 0, b == 0), (l1, l2, l3)


def test_real_cg_rejects_bad_triples():
    with pytest.raises(C.CgtpError) as e:
        C.real_cg(1, 1, 3)
    assert e.value.status == 6


@pytest.mark.parametrize("name", ["tiny", "lmax2", "lmax2_wide", "lmax3"])
def test_neighbor_list_bit_exact(name):
    c = WL.CONFIGS[name]
    pos, box = WL.si_diamond(c["cells"], c["sigma"], 0)
    rp_o, col_o, sh_o, vec_o = O.neighbor_list(pos, box, c["rc"])
    rp, col, sh, r = C.neighbor_list(pos, box, c["rc"])
    assert np.array_equal(rp.astype(np.int64), rp_o)
    assert np.array_equal(col, col_o)
    assert np.array_equal(sh, sh_o)
    assert np.array_equal(r, vec_o.astype(np.float32))


@pytest.mark.parametrize("cells,rc", [((1, 1, 1), 5.0), ((1, 1, 2), 6.0), ((2, 1, 1), 11.0)])
def test_neighbor_list_small_boxes_many_images(cells, rc):
    pos, box = WL.si_diamond(cells, 0.07, 3)
    rp_o, col_o, sh_o, vec_o = O.neighbor_list(pos, box, rc)
    rp, col, sh, r = C.neighbor_list(pos, box, rc)
    assert np.array_equal(rp.astype(np.int64), rp_o) and np.array_equal(col, col_o)
    assert np.array_equal(sh, sh_o) and np.array_equal(r, vec_o.astype(np.float32))


@pytest.mark.parametrize("threads", ["1", "3", "7"])
def test_neighbor_list_independent_of_host_threads(threads, monkeypatch):
    """Receivers split over host threads (uneven ranges here) give the
    oracle's brute-force list bit for bit."""
    pos, box = WL.si_diamond((2, 2, 3), 0.07, 4)
    rp_o, col_o, sh_o, vec_o = O.neighbor_list(pos, box, 5.0)
    monkeypatch.setenv("CGTP_HOST_THREADS", threads)
    rp, col, sh, r = C.neighbor_list(pos, box, 5.0)
    assert np.array_equal(rp.astype(np.int64), rp_o) and np.array_equal(col, col_o)
    assert np.array_equal(sh, sh_o) and np.array_equal(r, vec_o.astype(np.float32))


def test_neighbor_list_rejects_unwrapped_positions():
    with pytest.raises(C.CgtpError):
        C.neighbor_list(np.array([[0.0, 0.0, 5.0]]), np.array([4.0, 4.0, 4.0]), 3.0)


def test_csr_transpose():
    rng = np.random.default_rng(1)
    deg = rng.integers(0, 6, size=40)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    col = rng.integers(0, 25, size=rowptr[-1]).astype(np.int32)
    rpt, perm = C.csr_transpose(rowptr, col, 25)
    assert rpt[0] == 0 and rpt[-1] == len(col)
    for j in range(25):
        ids = perm[rpt[j]:rpt[j + 1]]
        assert np.all(col[ids] == j) and np.all(np.diff(ids) > 0)
    assert np.array_equal(np.sort(perm), np.arange(len(col)))
    with pytest.raises(C.CgtpError):
        C.csr_transpose(rowptr, np.full_like(col, 30), 25)


@pytest.fixture
def compile_only(monkeypatch):
    monkeypatch.setenv("CGTP_JIT_COMPILE_ONLY", "1")


@pytest.mark.parametrize("name", ["tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6", "case4", "case5", "case6"])
def test_plan_builds_and_compiles(name, compile_only):
    c = WL.CONFIGS[name]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    assert (plan.d_in, plan.d_edge, plan.d_out, plan.n_weights, plan.n_paths) == \
        (P.D_in, P.D_e, P.D_out, P.U, P.npaths)
    assert np.array_equal(plan.paths(), P.table)
    assert np.allclose(plan.coefficients(), P.cg, atol=1e-12)
    text = plan.describe()
    assert "cgtp_fwd" in text and "cgtp_bwd" in text
    # a compile-only plan refuses to launch
    with pytest.raises(C.CgtpError):
        plan.check_device_error()


@pytest.mark.parametrize("args,status", [
    (("16x0e+", "1x0e", "16x0e"), 3),
    (("16x0e", "1x0e+1x2e", "16x0e"), 3),
    (("16x0e+16x1o", "1x0e+1x1o", "32x0e+16x1o"), 4),
    (("16x7e", "1x0e", "16x7e"), 5),
])
def test_plan_argument_errors(args, status, compile_only):
    with pytest.raises(C.CgtpError) as e:
        C.Plan(*args, 6)
    assert e.value.status == status


def test_lmax_bound(compile_only):
    with pytest.raises(C.CgtpError) as e:
        C.Plan("4x3e", "1x0e+1x1o", "4x3e+4x2o+4x4o", 2)
    assert e.value.status == 5


def test_force_chain_argument_errors(compile_only):
    """cgtp_sph_harm_backward / cgtp_edge_forces / cgtp_edge_virial validate
    before any launch."""
    OK, NULL, ALIGN, SIZE = 0, 1, 2, 6  # cgtp_status codes of include/cgtp.h
    lib = C._lib
    plan = C.Plan("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", 6)
    assert lib.cgtp_sph_harm_backward(None, 1, None, None, None, None) == NULL
    assert lib.cgtp_sph_harm_backward(plan._h, -1, None, None, None, None) == SIZE
    assert lib.cgtp_sph_harm_backward(plan._h, 4, None, None, None, None) == NULL
    assert lib.cgtp_sph_harm_backward(plan._h, 0, None, None, None, None) == OK  # nothing to do
    assert lib.cgtp_edge_forces(-1, 0, None, None, None, None, None, None) == SIZE
    assert lib.cgtp_edge_forces(0, 0, None, None, None, None, None, None) == OK
    assert lib.cgtp_edge_forces(4, 8, None, None, None, None, None, None) == NULL
    p16, p4 = ctypes.c_void_p(16), ctypes.c_void_p(4)  # never dereferenced: refused first
    assert lib.cgtp_edge_virial(-1, None, None, p16, None) == SIZE
    assert lib.cgtp_edge_virial(1 << 31, p16, p16, p16, None) == SIZE
    assert lib.cgtp_edge_virial(4, p16, p16, None, None) == NULL
    assert lib.cgtp_edge_virial(4, None, p16, p16, None) == NULL
    assert lib.cgtp_edge_virial(4, p16, None, p16, None) == NULL
    assert lib.cgtp_edge_virial(4, p4, p16, p16, None) == ALIGN
    assert lib.cgtp_edge_virial(4, p16, p4, p16, None) == ALIGN


def test_binding_checks_tensors_before_the_abi(compile_only):
    """The binding refuses a tensor whose dtype, element count or device
    would let a kernel's flat indexing leave it, before any pointer crosses
    the C ABI (checked in that order, so CPU tensors reach each check)."""
    torch = pytest.importorskip("torch")
    plan = C.Plan("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", 6)
    n, E = 3, 5
    rowptr = torch.tensor([0, 2, 4, 5], dtype=torch.int32)
    col = torch.tensor([1, 2, 0, 2, 1], dtype=torch.int32)
    x = torch.zeros(n, plan.d_in)
    Y = torch.zeros(E, plan.d_edge)
    W = torch.zeros(E, plan.n_weights)
    with pytest.raises(TypeError, match="x: expected torch.float32"):
        plan.forward(rowptr, col, x.double(), Y, W)
    with pytest.raises(TypeError, match="rowptr: expected torch.int32"):
        plan.forward(rowptr.long(), col, x, Y, W)
    with pytest.raises(ValueError, match="W: expected"):
        plan.forward(rowptr, col, x, Y, W[:, 1:].contiguous())
    with pytest.raises(ValueError, match="out: expected"):
        plan.forward(rowptr, col, x, Y, W, out=torch.zeros(n, plan.d_out - 1))
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        plan.forward(rowptr, col, x, Y, W)
    g = torch.zeros(n, plan.d_out)
    with pytest.raises(ValueError, match="rowptr_T: expected"):
        plan.backward(rowptr, col, rowptr[:-1].contiguous(), col, x, Y, W, g)
    with pytest.raises(ValueError, match="grad_out: expected"):
        plan.backward(rowptr, col, rowptr, col, x, Y, W, g[:-1])
    r = torch.zeros(E, 3)
    with pytest.raises(ValueError, match="grad_Y: expected"):
        plan.sph_harm_backward(r, torch.zeros(E, plan.d_edge + 1))
    with pytest.raises(TypeError, match="r: expected torch.float32"):
        C.edge_virial(r.int(), r)
    with pytest.raises(ValueError, match="grad_r: expected"):
        C.edge_virial(r, r[:-1])
    with pytest.raises(ValueError, match="perm_T: expected"):
        C.edge_forces(rowptr, rowptr, col[:-1], r)


def test_double_backward_host_checks(compile_only):
    torch = pytest.importorskip("torch")
    NULL, SIZE = 1, 6
    lib = C._lib
    plan = C.Plan("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", 6)
    args = [None] * 16 + [0, None]
    assert lib.cgtp_double_backward(None, 1, 1, 1, *args) == NULL
    assert lib.cgtp_double_backward(plan._h, -1, 1, 1, *args) == SIZE
    # the workspace holds the backward's and one scratch row set per output
    n_recv, n_send, E = 7, 5, 40
    need = plan.double_backward_workspace_size(n_recv, n_send, E)
    floats = n_recv * plan.d_out + n_send * plan.d_in + E * plan.n_weights + E * plan.d_edge
    assert need >= plan.workspace_size(n_recv, n_send, E) + 4 * floats
    assert plan.double_backward_workspace_size(n_recv, n_send, 2 * E) > need
    # the binding checks the cotangents like every other tensor
    rowptr = torch.tensor([0, 2, 4, 5], dtype=torch.int32)
    col = torch.tensor([1, 2, 0, 2, 1], dtype=torch.int32)
    x, Y, W = torch.zeros(3, plan.d_in), torch.zeros(5, plan.d_edge), torch.zeros(5, plan.n_weights)
    g = torch.zeros(3, plan.d_out)
    with pytest.raises(ValueError, match="h_W: expected"):
        plan.double_backward(rowptr, col, rowptr, col, x, Y, W, g, h_W=W[:4])
    with pytest.raises(TypeError, match="h_Y: expected torch.float32"):
        plan.double_backward(rowptr, col, rowptr, col, x, Y, W, g, h_Y=Y.double())


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_is_plain_c(lang, std, tmp_path):
    """include/cgtp.h compiles on its own as strict C99 and as C++11 (no CUDA
    or torch headers needed by a caller of the C ABI)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "cgtp.h"\n'
                   "static cgtp_status (*destroy)(cgtp_plan) = cgtp_plan_destroy;\n"
                   "static const char* (*name)(cgtp_status) = cgtp_status_string;\n"
                   "int main(void) { return destroy(0) != CGTP_OK || name(CGTP_OK) == 0; }\n")
    p = subprocess.run([cc, "-x", lang, std, "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.dirname(HEADER), "-c", str(src), "-o", str(tmp_path / "use.o")],
                       capture_output=True, text=True)
    assert p.returncode == 0, p.stderr


C_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include "cgtp.h"
int main(void) {
  /* one diamond-cubic cell (a = 5.43): every atom has 4 neighbours within 2.5 */
  const double a = 5.43, box[3] = {5.43, 5.43, 5.43};
  const double f[8][3] = {{0, 0, 0}, {0, .5, .5}, {.5, 0, .5}, {.5, .5, 0},
                          {.25, .25, .25}, {.25, .75, .75}, {.75, .25, .75}, {.75, .75, .25}};
  double pos[24];
  for (int i = 0; i < 24; ++i) pos[i] = a * f[i / 3][i % 3];
  int32_t rowptr[9], rpt[9];
  int64_t E = 0;
  if (cgtp_neighbor_list(8, pos, box, 2.5, rowptr, NULL, NULL, NULL, &E) != CGTP_OK) return 1;
  int32_t* col = malloc(sizeof(int32_t) * E);
  int32_t* perm = malloc(sizeof(int32_t) * E);
  float* r = malloc(sizeof(float) * 3 * E);
  if (cgtp_neighbor_list(8, pos, box, 2.5, rowptr, col, NULL, r, &E) != CGTP_OK) return 2;
  if (cgtp_csr_transpose(8, 8, E, rowptr, col, rpt, perm) != CGTP_OK) return 3;
  cgtp_plan plan = NULL;
  if (cgtp_plan_create("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", 6, &plan) != CGTP_OK) {
    fprintf(stderr, "%s\n", cgtp_last_error());
    return 4;
  }
  int64_t din, de, dout, nw, np;
  cgtp_plan_info(plan, &din, &de, &dout, &nw, &np);
  printf("E=%lld rpt8=%d din=%lld de=%lld dout=%lld nw=%lld paths=%lld\n", (long long)E, rpt[8],
         (long long)din, (long long)de, (long long)dout, (long long)nw, (long long)np);
  cgtp_status bad = cgtp_plan_create("16x0e+", "1x0e", "16x0e", 6, &plan);
  printf("bad=%s\n", cgtp_status_string(bad));
  free(col);
  free(perm);
  free(r);
  return 0;
}
"""


def test_c_program_uses_the_abi(tmp_path):
    """A C program linked against libcgtp.so alone (no Python, no torch)
    builds a neighbour list and its transpose and a compile-only plan."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no host compiler")
    from equivariant_mlip_clebsch_b200 import build as B
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "prog"
    libdir = os.path.dirname(B.LIB)
    p = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o",
                        str(exe), "-L", libdir, "-lcgtp", "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert p.returncode == 0, p.stderr
    env = dict(os.environ, CGTP_JIT_COMPILE_ONLY="1", CGTP_JIT_CACHE=str(tmp_path / "cache"))
    run = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=600)
    assert run.returncode == 0, run.stderr
    assert run.stdout.splitlines() == ["E=32 rpt8=32 din=64 de=4 dout=128 nw=64 paths=4",
                                       "bad=CGTP_ERR_IRREPS_PARSE"]


def test_header_error_lists_name_real_statuses():
    """Every status an entry's "Errors:" list names exists in cgtp_status."""
    text = open(HEADER).read()
    enum = set(re.findall(r"CGTP_ERR_(\w+)\s*=", text))
    lists = re.findall(r"Errors:\s*([A-Z_, ]+)", text)
    assert lists
    for lst in lists:
        for name in re.findall(r"[A-Z][A-Z_]+", lst):
            assert name in enum, (name, lst)


COMPOSE_HOST = r"""
#include <cstdint>
#include <vector>
#include "double_backward.hpp"
extern "C" {
void orc_forward(int64_t, const int64_t*, const int32_t*, int, int, int, int, const double*, const double*,
                 const double*, int, const int32_t*, const double*, double*, int);
void orc_backward(int64_t, int64_t, int64_t, const int64_t*, const int32_t*, int, int, int, int, const double*,
                  const double*, const double*, const double*, int, const int32_t*, const double*, double*,
                  double*, double*, int);
}
struct HostOps {  // the oracle's forward and backward on host buffers
  cgtp::DbwdDims d;
  const int64_t* rowptr;
  const int32_t* col;
  int npaths;
  const int32_t* paths;
  const double* cg;
  const float* g;
  static std::vector<double> up(const float* p, int64_t n) { return std::vector<double>(p, p + n); }
  static void down(const std::vector<double>& v, float* p) {
    for (size_t i = 0; i < v.size(); ++i) p[i] = (float)v[i];
  }
  int forward(const float* x, const float* Y, const float* W, float* out) {
    auto xd = up(x, d.n_send * d.D_in), yd = up(Y, d.E * d.D_e), wd = up(W, d.E * d.U);
    std::vector<double> o(d.n_recv * d.D_out);
    orc_forward(d.n_recv, rowptr, col, (int)d.D_in, (int)d.D_e, (int)d.D_out, (int)d.U, xd.data(), yd.data(),
                wd.data(), npaths, paths, cg, o.data(), 0);
    down(o, out);
    return 0;
  }
  int backward(const float* x, const float* Y, const float* W, float* ox, float* ow, float* oy) {
    auto xd = up(x, d.n_send * d.D_in), yd = up(Y, d.E * d.D_e), wd = up(W, d.E * d.U);
    auto gd = up(g, d.n_recv * d.D_out);
    std::vector<double> vx(ox ? d.n_send * d.D_in : 0), vw(ow ? d.E * d.U : 0), vy(oy ? d.E * d.D_e : 0);
    orc_backward(d.n_recv, d.n_send, d.E, rowptr, col, (int)d.D_in, (int)d.D_e, (int)d.D_out, (int)d.U, xd.data(),
                 yd.data(), wd.data(), gd.data(), npaths, paths, cg, ox ? vx.data() : nullptr,
                 ow ? vw.data() : nullptr, oy ? vy.data() : nullptr, 0);
    if (ox) down(vx, ox);
    if (ow) down(vw, ow);
    if (oy) down(vy, oy);
    return 0;
  }
  int add(float* dst, const float* src, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] += src[i];
    return 0;
  }
  int zero(float* dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] = 0.f;
    return 0;
  }
};
extern "C" int run_compose(const int64_t* dims, const int64_t* rowptr, const int32_t* col, int npaths,
                           const int32_t* paths, const double* cg, const float* x, const float* Y, const float* W,
                           const float* g, const float* h_x, const float* h_W, const float* h_Y, float* gg,
                           float* gx, float* gW, float* gY) {
  const cgtp::DbwdDims d{dims[0], dims[1], dims[2], dims[3], dims[4], dims[5], dims[6]};
  std::vector<float> tF(d.n_recv * d.D_out), tX(d.n_send * d.D_in), tW(d.E * d.U), tY(d.E * d.D_e);
  HostOps ops{d, rowptr, col, npaths, paths, cg, g};
  return cgtp::compose_double_backward(ops, d, x, Y, W, h_x, h_W, h_Y, gg, gx, gW, gY, tF.data(), tX.data(),
                                       tW.data(), tY.data());
}
"""


@pytest.mark.parametrize("keys", [(), ("h_x",), ("h_W",), ("h_Y",), ("h_x", "h_W"), ("h_W", "h_Y"),
                                  ("h_x", "h_Y"), ("h_x", "h_W", "h_Y")])
def test_double_backward_composition_on_host(keys, tmp_path):
    """The library's double-backward term structure (csrc/double_backward.hpp,
    the code cgtp_double_backward runs on the kernels) driven by the oracle's
    forward and backward on the host equals the oracle's own composition:
    which term writes an output in place, which adds through scratch, which
    output is zeroed.  Outputs start as NaN; two are left out in one case."""
    import ctypes
    import shutil
    import subprocess
    if shutil.which("g++") is None:
        pytest.skip("no host compiler")
    src = tmp_path / "compose.cpp"
    src.write_text(COMPOSE_HOST)
    so = tmp_path / "libcompose.so"
    orc = O.build()
    csrc = os.path.join(os.path.dirname(os.path.dirname(__file__)), "equivariant_mlip_clebsch_b200", "csrc")
    p = subprocess.run(["g++", "-std=c++17", "-O1", "-shared", "-fPIC", "-I", csrc, str(src), "-o", str(so),
                        orc, "-Wl,-rpath," + os.path.dirname(orc)], capture_output=True, text=True)
    assert p.returncode == 0, p.stderr
    lib = ctypes.CDLL(str(so))
    rng = np.random.default_rng(5)
    P = O.enumerate_paths("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o")
    n_recv, n_send = 7, 6
    deg = rng.integers(0, 5, size=n_recv)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    E = int(rowptr[-1])
    col = rng.integers(0, n_send, size=E).astype(np.int32)
    f32 = lambda *s: rng.standard_normal(s).astype(np.float32)
    x, Y, W, g = f32(n_send, P.D_in), f32(E, P.D_e), f32(E, P.U), f32(n_recv, P.D_out)
    h = {"h_x": f32(n_send, P.D_in), "h_W": f32(E, P.U), "h_Y": f32(E, P.D_e)}
    h = {k: (v if k in keys else None) for k, v in h.items()}
    want = {"gg": (n_recv, P.D_out), "gx": (n_send, P.D_in), "gW": (E, P.U), "gY": (E, P.D_e)}
    skip = {"gx", "gY"} if keys == ("h_x", "h_W") else set()  # outputs not asked for
    outs = {k: (None if k in skip else np.full(s, np.nan, dtype=np.float32)) for k, s in want.items()}
    ptr = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    dims = np.array([n_recv, n_send, E, P.D_in, P.D_e, P.D_out, P.U], dtype=np.int64)
    table = np.ascontiguousarray(P.table, dtype=np.int32)
    cg = np.ascontiguousarray(P.cg, dtype=np.float64)
    lib.run_compose.restype = ctypes.c_int
    rc = lib.run_compose(ptr(dims), ptr(rowptr), ptr(col), ctypes.c_int(P.npaths), ptr(table), ptr(cg), ptr(x),
                         ptr(Y), ptr(W), ptr(g), ptr(h["h_x"]), ptr(h["h_W"]), ptr(h["h_Y"]), ptr(outs["gg"]),
                         ptr(outs["gx"]), ptr(outs["gW"]), ptr(outs["gY"]))
    assert rc == 0
    ref = O.double_backward(P, rowptr, col, n_send, x, Y, W, g, **h)
    for k, r in zip(("gg", "gx", "gW", "gY"), ref):
        if outs[k] is None:
            continue
        assert np.isfinite(outs[k]).all(), k
        assert np.allclose(outs[k], r, rtol=1e-5, atol=1e-5 * max(1.0, np.abs(r).max())), k
