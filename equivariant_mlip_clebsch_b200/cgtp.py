"""Python binding of libcgtp (include/cgtp.h): argument checks and
marshalling only.

Every step of the convolution runs in the library's CUDA kernels; torch is used
for device memory and the current stream.  Each tensor's dtype, element count
and device are checked before its pointer crosses the ABI.  There is no
fallback: if the library is missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_PKG = os.path.dirname(os.path.abspath(__file__))
if os.environ.setdefault("CGTP_JIT_CACHE", os.path.join(_PKG, "_jit_cache")):
    os.makedirs(os.environ["CGTP_JIT_CACHE"], exist_ok=True)

if not os.path.exists(_build.LIB):
    raise ImportError(f"{_build.LIB} is not built; run equivariant_mlip_clebsch_b200.build.build()")

_lib = ctypes.CDLL(_build.LIB)

_P, _i, _i64, _d, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
_pi64 = ctypes.POINTER(ctypes.c_int64)

_SIGS = {
    "cgtp_status_string": (ctypes.c_char_p, [_i]),
    "cgtp_last_error": (ctypes.c_char_p, []),
    "cgtp_plan_create": (_i, [ctypes.c_char_p, ctypes.c_char_p, ctypes.c_char_p, _i,
                              ctypes.POINTER(_P)]),
    "cgtp_plan_destroy": (_i, [_P]),
    "cgtp_plan_info": (_i, [_P, _pi64, _pi64, _pi64, _pi64, _pi64]),
    "cgtp_plan_paths": (_i, [_P, _P]),
    "cgtp_plan_coefficients": (_i, [_P, _P, _pi64]),
    "cgtp_plan_describe": (_i, [_P, ctypes.c_char_p, _sz, ctypes.POINTER(_sz)]),
    "cgtp_real_cg": (_i, [_i, _i, _i, _P]),
    "cgtp_sph_harm": (_i, [_P, _i64, _P, _P, _P]),
    "cgtp_sph_harm_backward": (_i, [_P, _i64, _P, _P, _P, _P]),
    "cgtp_edge_forces": (_i, [_i64, _i64, _P, _P, _P, _P, _P, _P]),
    "cgtp_edge_virial": (_i, [_i64, _P, _P, _P, _P]),
    "cgtp_double_backward_workspace_size": (_i, [_P, _i64, _i64, _i64, ctypes.POINTER(_sz)]),
    "cgtp_double_backward": (_i, [_P, _i64, _i64, _i64] + [_P] * 16 + [_sz, _P]),
    "cgtp_plan_prepare_double_backward": (_i, [_P, ctypes.POINTER(_i)]),
    "cgtp_forward": (_i, [_P, _i64, _i64, _i64, _P, _P, _P, _P, _P, _P, _P]),
    "cgtp_backward_workspace_size": (_i, [_P, _i64, _i64, _i64, ctypes.POINTER(_sz)]),
    "cgtp_backward": (_i, [_P, _i64, _i64, _i64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                           _P, _sz, _P]),
    "cgtp_backward_static_scratch": (_i, [_P, _i64, _i64, _i64, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          _P, _P, _P]),
    "cgtp_plan_check_device_error": (_i, [_P, ctypes.POINTER(_i)]),
    "cgtp_plan_set_timing": (_i, [_P, _i]),
    "cgtp_plan_set_checks": (_i, [_P, _i]),
    "cgtp_validate_graph": (_i, [_P, _i64, _i64, _i64, _P, _P, _P, _P, _P]),
    "cgtp_plan_kernel_times": (_i, [_P, _i, ctypes.c_char_p, _P, _P, ctypes.POINTER(_i)]),
    "cgtp_sparse_workspace_size": (_i, [_P, _i64, _i64, _i64, ctypes.POINTER(_sz)]),
    "cgtp_sparse_forward": (_i, [_P, _i64, _i64, _i64] + [_P] * 8 + [_sz, _P]),
    "cgtp_sparse_backward": (_i, [_P, _i64, _i64, _i64] + [_P] * 14 + [_sz, _P]),
    "cgtp_fma_peak_sink_floats": (_i, [_pi64]),
    "cgtp_fma_peak": (_i, [_i64, _P, _i64, _P, ctypes.POINTER(_d)]),
    "cgtp_neighbor_list": (_i, [_i64, _P, _P, _d, _P, _P, _P, _P, _pi64]),
    "cgtp_csr_transpose": (_i, [_i64, _i64, _i64, _P, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTS = tuple(_SIGS)
STATIC_SCRATCH_BYTES = 64 << 20  # CGTP_STATIC_SCRATCH_BYTES of include/cgtp.h


class CgtpError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


def _check(st: int) -> None:
    if st != 0:
        raise CgtpError(st, _lib.cgtp_last_error().decode())


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _require_device(t, name, dev):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor")
    if dev is not None and t.device != dev:
        raise ValueError(f"{name}: on {t.device}, the other arguments on {dev}")


def _args(dev, *specs):
    """Device pointers of tensor arguments, each spec (tensor, name, count,
    kind), after the checks that keep the kernels' flat indexing inside
    them: first dtype (kind "f32" or "i32") and exactly `count` elements for
    every argument, then a contiguous CUDA tensor on `dev`.  None passes as
    NULL (the library then reports a required argument as CGTP_ERR_NULL)."""
    import torch
    for t, name, count, kind in specs:
        if t is None:
            continue
        want = torch.float32 if kind == "f32" else torch.int32
        if t.dtype != want:
            raise TypeError(f"{name}: expected {want}, got {t.dtype}")
        if t.numel() != count:
            raise ValueError(f"{name}: expected {count} elements, got shape {tuple(t.shape)}")
    for t, name, _, _ in specs:
        if t is not None:
            _require_device(t, name, dev)
    return [None if t is None else ctypes.c_void_p(t.data_ptr()) for t, _, _, _ in specs]


def _workspace(t, dev):
    """Pointer and byte size of a caller workspace (any dtype)."""
    _require_device(t, "workspace", dev)
    return ctypes.c_void_p(t.data_ptr()), t.numel() * t.element_size()


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1), dtype=np.float64)
    _check(_lib.cgtp_real_cg(l1, l2, l3, _np_ptr(C)))
    return C


def neighbor_list(pos, box, rc: float):
    """Cell-list neighbour list (host).  Returns rowptr, col, shift (int32)
    and the FP32 edge vectors r = pos_j + n*box - pos_i."""
    pos = np.ascontiguousarray(pos, dtype=np.float64)
    box = np.ascontiguousarray(box, dtype=np.float64)
    N = pos.shape[0]
    rowptr = np.zeros(N + 1, dtype=np.int32)
    E = ctypes.c_int64(0)
    _check(_lib.cgtp_neighbor_list(N, _np_ptr(pos), _np_ptr(box), float(rc), _np_ptr(rowptr),
                                   None, None, None, ctypes.byref(E)))
    col = np.zeros(E.value, dtype=np.int32)
    shift = np.zeros((E.value, 3), dtype=np.int32)
    r = np.zeros((E.value, 3), dtype=np.float32)
    _check(_lib.cgtp_neighbor_list(N, _np_ptr(pos), _np_ptr(box), float(rc), _np_ptr(rowptr),
                                   _np_ptr(col), _np_ptr(shift), _np_ptr(r), ctypes.byref(E)))
    return rowptr, col, shift, r


def edge_forces(rowptr, rowptr_T, perm_T, grad_r, forces=None, stream=None):
    """cgtp_edge_forces: forces [N,3] = -dL/dpos from grad_r [E,3] (device
    tensors; r_e = pos_sender - pos_receiver + shift)."""
    import torch
    n_atoms, E, dev = rowptr.shape[0] - 1, grad_r.shape[0], grad_r.device
    if forces is None:
        forces = torch.empty((n_atoms, 3), dtype=torch.float32, device=dev)
    ptrs = _args(dev, (rowptr, "rowptr", n_atoms + 1, "i32"), (rowptr_T, "rowptr_T", n_atoms + 1, "i32"),
                 (perm_T, "perm_T", E, "i32"), (grad_r, "grad_r", 3 * E, "f32"),
                 (forces, "forces", 3 * n_atoms, "f32"))
    _check(_lib.cgtp_edge_forces(n_atoms, E, *ptrs, _stream(stream)))
    return forces


def edge_virial(r, grad_r, virial=None, stream=None):
    """cgtp_edge_virial: the strain derivative V [3,3], V[a,b] = sum_e
    grad_r[e,a] r[e,b] (device tensors; stress = V / cell volume)."""
    import torch
    E, dev = r.shape[0], r.device
    if virial is None:
        virial = torch.empty((3, 3), dtype=torch.float32, device=dev)
    ptrs = _args(dev, (r, "r", 3 * E, "f32"), (grad_r, "grad_r", 3 * E, "f32"), (virial, "virial", 9, "f32"))
    _check(_lib.cgtp_edge_virial(E, *ptrs, _stream(stream)))
    return virial


def csr_transpose(rowptr, col, n_send: int):
    rowptr = np.ascontiguousarray(rowptr, dtype=np.int32)
    col = np.ascontiguousarray(col, dtype=np.int32)
    n_recv, E = rowptr.shape[0] - 1, col.shape[0]
    rowptr_T = np.zeros(n_send + 1, dtype=np.int32)
    perm_T = np.zeros(max(E, 1), dtype=np.int32)
    _check(_lib.cgtp_csr_transpose(n_recv, n_send, E, _np_ptr(rowptr), _np_ptr(col),
                                   _np_ptr(rowptr_T), _np_ptr(perm_T)))
    return rowptr_T, perm_T[:E]


class Plan:
    """A CGTP plan: irreps, paths, CG tables and the compiled kernels."""

    def __init__(self, irreps_in: str, irreps_edge: str, irreps_out: str, lmax: int | None = None):
        if lmax is None:
            lmax = 6
        h = ctypes.c_void_p()
        _check(_lib.cgtp_plan_create(irreps_in.encode(), irreps_edge.encode(), irreps_out.encode(),
                                     int(lmax), ctypes.byref(h)))
        self._h = h
        self.irreps_in, self.irreps_edge, self.irreps_out = irreps_in, irreps_edge, irreps_out
        v = [ctypes.c_int64() for _ in range(5)]
        _check(_lib.cgtp_plan_info(h, *[ctypes.byref(t) for t in v]))
        self.d_in, self.d_edge, self.d_out, self.n_weights, self.n_paths = (t.value for t in v)
        self.L = int(round(self.d_edge ** 0.5)) - 1

    def close(self):
        if getattr(self, "_h", None):
            _lib.cgtp_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- host introspection
    def paths(self) -> np.ndarray:
        t = np.zeros((self.n_paths, 8), dtype=np.int32)
        if self.n_paths:
            _check(_lib.cgtp_plan_paths(self._h, _np_ptr(t)))
        return t

    def coefficients(self) -> np.ndarray:
        n = ctypes.c_int64()
        _check(_lib.cgtp_plan_coefficients(self._h, None, ctypes.byref(n)))
        c = np.zeros(n.value, dtype=np.float64)
        _check(_lib.cgtp_plan_coefficients(self._h, _np_ptr(c), ctypes.byref(n)))
        return c

    def describe(self) -> str:
        need = ctypes.c_size_t()
        _check(_lib.cgtp_plan_describe(self._h, None, 0, ctypes.byref(need)))
        buf = ctypes.create_string_buffer(need.value)
        _check(_lib.cgtp_plan_describe(self._h, buf, need.value, ctypes.byref(need)))
        return buf.value.decode()

    def out_fan_in(self) -> list:
        """Number of paths feeding each output irrep block (in order)."""
        muls = [int(tok.split("x")[0]) for tok in self.irreps_out.split("+")]
        base = np.concatenate([[0], np.cumsum(muls)])
        fan = [0] * len(muls)
        for k0 in self.paths()[:, 5]:
            fan[int(np.searchsorted(base, k0, side="right")) - 1] += 1
        return fan

    def check_device_error(self) -> None:
        code = ctypes.c_int()
        _check(_lib.cgtp_plan_check_device_error(self._h, ctypes.byref(code)))

    def set_checks(self, enable: bool) -> None:
        """cgtp_plan_set_checks: device checks of the graph before every call
        (each call then waits for their result)."""
        _check(_lib.cgtp_plan_set_checks(self._h, 1 if enable else 0))

    def validate_graph(self, rowptr, col, n_send: int, rowptr_T=None, perm_T=None, stream=None) -> None:
        """cgtp_validate_graph: the device graph checks once, whatever the
        plan's flags (raises CgtpError with status 7 naming the failed
        checks)."""
        if (rowptr_T is None) != (perm_T is None):
            raise ValueError("rowptr_T and perm_T go together")
        n_recv, E, dev = rowptr.shape[0] - 1, col.shape[0], rowptr.device
        ptrs = _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (rowptr_T, "rowptr_T", n_send + 1, "i32"), (perm_T, "perm_T", E, "i32"))
        _check(_lib.cgtp_validate_graph(self._h, n_recv, n_send, E, *ptrs, _stream(stream)))

    def set_timing(self, enable: bool) -> None:
        _check(_lib.cgtp_plan_set_timing(self._h, int(bool(enable))))

    def kernel_times(self) -> dict:
        """{kernel name: (total ms, launches)} since the previous call."""
        mx = 16
        names = ctypes.create_string_buffer(32 * mx)
        ms = np.zeros(mx, dtype=np.float64)
        cnt = np.zeros(mx, dtype=np.int64)
        n = ctypes.c_int()
        _check(_lib.cgtp_plan_kernel_times(self._h, mx, names, _np_ptr(ms), _np_ptr(cnt), ctypes.byref(n)))
        out = {}
        for k in range(min(n.value, mx)):
            nm = names.raw[32 * k:32 * (k + 1)].split(b"\0", 1)[0].decode()
            out[nm] = (float(ms[k]), int(cnt[k]))
        return out

    # ---- device calls
    def sph_harm(self, r, Y=None, stream=None):
        import torch
        E, dev = r.shape[0], r.device
        if Y is None:
            Y = torch.empty((E, self.d_edge), dtype=torch.float32, device=dev)
        ptrs = _args(dev, (r, "r", 3 * E, "f32"), (Y, "Y", E * self.d_edge, "f32"))
        _check(_lib.cgtp_sph_harm(self._h, E, *ptrs, _stream(stream)))
        return Y

    def sph_harm_backward(self, r, grad_Y, grad_r=None, stream=None):
        """cgtp_sph_harm_backward: grad_r [E,3] = sum_t grad_Y[:, t] dY_t/dr."""
        import torch
        E, dev = r.shape[0], r.device
        if grad_r is None:
            grad_r = torch.empty((E, 3), dtype=torch.float32, device=dev)
        ptrs = _args(dev, (r, "r", 3 * E, "f32"), (grad_Y, "grad_Y", E * self.d_edge, "f32"),
                     (grad_r, "grad_r", 3 * E, "f32"))
        _check(_lib.cgtp_sph_harm_backward(self._h, E, *ptrs, _stream(stream)))
        return grad_r

    def forward(self, rowptr, col, x, Y, W, out=None, stream=None):
        import torch
        n_recv, n_send, E, dev = rowptr.shape[0] - 1, x.shape[0], col.shape[0], x.device
        if out is None:
            out = torch.empty((n_recv, self.d_out), dtype=torch.float32, device=dev)
        ptrs = _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (x, "x", n_send * self.d_in, "f32"), (Y, "Y", E * self.d_edge, "f32"),
                     (W, "W", E * self.n_weights, "f32"), (out, "out", n_recv * self.d_out, "f32"))
        _check(_lib.cgtp_forward(self._h, n_recv, n_send, E, *ptrs, _stream(stream)))
        return out

    def _grads(self, want, grads, n_send, E, dev):
        """The caller's (dx, dW, dY), or new tensors for the gradients in `want`."""
        if grads is not None:
            return grads
        import torch
        f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
        return (f(n_send, self.d_in) if "x" in want else None,
                f(E, self.n_weights) if "W" in want else None,
                f(E, self.d_edge) if "Y" in want else None)

    def _backward_args(self, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out, dx, dW, dY, dev,
                       n_recv, n_send, E):
        return _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (rowptr_T, "rowptr_T", n_send + 1, "i32"), (perm_T, "perm_T", E, "i32"),
                     (x, "x", n_send * self.d_in, "f32"), (Y, "Y", E * self.d_edge, "f32"),
                     (W, "W", E * self.n_weights, "f32"), (grad_out, "grad_out", n_recv * self.d_out, "f32"),
                     (dx, "grad_x", n_send * self.d_in, "f32"), (dW, "grad_W", E * self.n_weights, "f32"),
                     (dY, "grad_Y", E * self.d_edge, "f32"))

    def workspace_size(self, n_recv: int, n_send: int, E: int) -> int:
        b = ctypes.c_size_t()
        _check(_lib.cgtp_backward_workspace_size(self._h, n_recv, n_send, E, ctypes.byref(b)))
        return b.value

    def backward(self, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out, want=("x", "W", "Y"),
                 grads=None, workspace=None, stream=None):
        import torch
        n_recv, n_send, E = rowptr.shape[0] - 1, x.shape[0], col.shape[0]
        dev = x.device
        dx, dW, dY = self._grads(want, grads, n_send, E, dev)
        if workspace is None:
            nbytes = self.workspace_size(n_recv, n_send, E)
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        _check(_lib.cgtp_backward(self._h, n_recv, n_send, E,
                                  *self._backward_args(rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out,
                                                       dx, dW, dY, dev, n_recv, n_send, E),
                                  *_workspace(workspace, dev), _stream(stream)))
        return dx, dW, dY

    def prepare_double_backward(self) -> bool:
        """cgtp_plan_prepare_double_backward: build the tangent kernels now;
        True when the double backward will use them."""
        t = ctypes.c_int()
        _check(_lib.cgtp_plan_prepare_double_backward(self._h, ctypes.byref(t)))
        return bool(t.value)

    def double_backward_workspace_size(self, n_recv: int, n_send: int, E: int) -> int:
        b = ctypes.c_size_t()
        _check(_lib.cgtp_double_backward_workspace_size(self._h, n_recv, n_send, E, ctypes.byref(b)))
        return b.value

    def double_backward(self, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out, h_x=None, h_W=None,
                        h_Y=None, want=("g", "x", "W", "Y"), grads=None, workspace=None, stream=None):
        """cgtp_double_backward: the gradients (d grad_out, dx, dW, dY) of
        S = <h_x, grad_x> + <h_W, grad_W> + <h_Y, grad_Y> over the backward
        at (x, Y, W, grad_out); None cotangents are zero."""
        import torch
        n_recv, n_send, E = rowptr.shape[0] - 1, x.shape[0], col.shape[0]
        dev = x.device
        if grads is None:
            f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
            grads = (f(n_recv, self.d_out) if "g" in want else None,
                     f(n_send, self.d_in) if "x" in want else None,
                     f(E, self.n_weights) if "W" in want else None,
                     f(E, self.d_edge) if "Y" in want else None)
        gg, gx, gW, gY = grads
        if workspace is None:
            nbytes = self.double_backward_workspace_size(n_recv, n_send, E)
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        ptrs = _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (rowptr_T, "rowptr_T", n_send + 1, "i32"), (perm_T, "perm_T", E, "i32"),
                     (x, "x", n_send * self.d_in, "f32"), (Y, "Y", E * self.d_edge, "f32"),
                     (W, "W", E * self.n_weights, "f32"), (grad_out, "grad_out", n_recv * self.d_out, "f32"),
                     (h_x, "h_x", n_send * self.d_in, "f32"), (h_W, "h_W", E * self.n_weights, "f32"),
                     (h_Y, "h_Y", E * self.d_edge, "f32"), (gg, "grad_grad_out", n_recv * self.d_out, "f32"),
                     (gx, "grad_x", n_send * self.d_in, "f32"), (gW, "grad_W", E * self.n_weights, "f32"),
                     (gY, "grad_Y", E * self.d_edge, "f32"))
        _check(_lib.cgtp_double_backward(self._h, n_recv, n_send, E, *ptrs, *_workspace(workspace, dev),
                                         _stream(stream)))
        return gg, gx, gW, gY

    # ---- BranchIP sparse evaluation (zero-gated edges skipped)
    def sparse_workspace_size(self, n_recv: int, n_send: int, E: int) -> int:
        b = ctypes.c_size_t()
        _check(_lib.cgtp_sparse_workspace_size(self._h, n_recv, n_send, E, ctypes.byref(b)))
        return b.value

    def _sparse_ws(self, workspace, n_recv, n_send, E, dev):
        if workspace is None:
            import torch
            workspace = torch.empty(max(self.sparse_workspace_size(n_recv, n_send, E), 256),
                                    dtype=torch.uint8, device=dev)
        return _workspace(workspace, dev)

    def sparse_forward(self, rowptr, col, x, Y, W, gate, out=None, workspace=None, stream=None):
        """cgtp_sparse_forward: out[i] = sum_e gate[e] TP_e over the edges with
        gate > 0 only (the full graph and full W, Y, gate are passed)."""
        import torch
        n_recv, n_send, E, dev = rowptr.shape[0] - 1, x.shape[0], col.shape[0], x.device
        if out is None:
            out = torch.empty((n_recv, self.d_out), dtype=torch.float32, device=dev)
        ptrs = _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (x, "x", n_send * self.d_in, "f32"), (Y, "Y", E * self.d_edge, "f32"),
                     (W, "W", E * self.n_weights, "f32"), (gate, "gate", E, "f32"),
                     (out, "out", n_recv * self.d_out, "f32"))
        _check(_lib.cgtp_sparse_forward(self._h, n_recv, n_send, E, *ptrs,
                                        *self._sparse_ws(workspace, n_recv, n_send, E, dev), _stream(stream)))
        return out

    def sparse_backward(self, rowptr, col, rowptr_T, perm_T, x, Y, W, gate, grad_out,
                        want=("x", "W", "Y", "gate"), grads=None, workspace=None, stream=None):
        """cgtp_sparse_backward: (dx, dW, dY, dgate) over the full edge set,
        zero on the skipped edges."""
        import torch
        n_recv, n_send, E, dev = rowptr.shape[0] - 1, x.shape[0], col.shape[0], x.device
        if grads is None:
            f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
            grads = (f(n_send, self.d_in) if "x" in want else None,
                     f(E, self.n_weights) if "W" in want else None,
                     f(E, self.d_edge) if "Y" in want else None,
                     f(E) if "gate" in want else None)
        dx, dW, dY, dg = grads
        ptrs = _args(dev, (rowptr, "rowptr", n_recv + 1, "i32"), (col, "col", E, "i32"),
                     (rowptr_T, "rowptr_T", n_send + 1, "i32"), (perm_T, "perm_T", E, "i32"),
                     (x, "x", n_send * self.d_in, "f32"), (Y, "Y", E * self.d_edge, "f32"),
                     (W, "W", E * self.n_weights, "f32"), (gate, "gate", E, "f32"),
                     (grad_out, "grad_out", n_recv * self.d_out, "f32"),
                     (dx, "grad_x", n_send * self.d_in, "f32"), (dW, "grad_W", E * self.n_weights, "f32"),
                     (dY, "grad_Y", E * self.d_edge, "f32"), (dg, "grad_gate", E, "f32"))
        _check(_lib.cgtp_sparse_backward(self._h, n_recv, n_send, E, *ptrs,
                                         *self._sparse_ws(workspace, n_recv, n_send, E, dev), _stream(stream)))
        return dx, dW, dY, dg

    def backward_static_scratch(self, rowptr, col, rowptr_T, perm_T, x, Y, W, grad_out,
                                want=("x", "W", "Y"), grads=None, stream=None):
        """cgtp_backward_static_scratch: the backward with the library's fixed
        device scratch instead of a workspace (no device allocation in the call
        when ``grads`` are given)."""
        n_recv, n_send, E = rowptr.shape[0] - 1, x.shape[0], col.shape[0]
        dev = x.device
        dx, dW, dY = self._grads(want, grads, n_send, E, dev)
        _check(_lib.cgtp_backward_static_scratch(self._h, n_recv, n_send, E,
                                                 *self._backward_args(rowptr, col, rowptr_T, perm_T, x, Y, W,
                                                                      grad_out, dx, dW, dY, dev, n_recv,
                                                                      n_send, E),
                                                 _stream(stream)))
        return dx, dW, dY
