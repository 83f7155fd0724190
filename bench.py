#!/usr/bin/env python
"""CGTP convolution throughput on B200.

One step = the whole hot path over one synthetic workload: real spherical
harmonics of the edge vectors, the forward CGTP convolution and its backward
(dL/dx, dL/dW, dL/dY).  The plan (paths, CG tables, kernel compilation) is
built once before timing.  Inputs are resident in HBM for ``value``; ``e2e``
repeats the step through the same public API with the inputs copied from
pinned host memory and the outputs copied back inside the timed region.
The headline is the Lmax=3 workload (6,144 atoms, the largest on one GPU);
``per_workload`` gives forward and forward+backward edges/s and atoms/s,
each kernel's fraction of its binding roof and the oracle's CPU rate for the
five workloads (tiny, lmax2, lmax2_wide, lmax3, lmax6).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
  python bench.py --impl reference ...     # the FP64 oracle on the host cores

Multi-GPU: the convolution is not sharded across GPUs; N ranks run N
independent replicas ("weak" scaling), timed on the device, max over ranks.
Prints one JSON line on rank 0 (details for humans go to stderr).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from equivariant_mlip_clebsch_b200 import workloads as WL  # noqa: E402

METRIC = "CGTP conv edges/s (fwd, fwd+bwd) on 1 B200; % of HBM/FP32 roofline"
# the headline workload: the largest that fits one GPU (Table 1 Case 3 on
# 6,144 atoms); the workloads of PER_WORKLOAD are measured beside it (the
# five of the target, then Table 1 Cases 4-6)
DEFAULT_CONFIG = "lmax3"
PER_WORKLOAD = ("tiny", "lmax2", "lmax2_wide", "lmax3", "lmax6", "case4", "case5", "case6")
L2_FLUSH_BYTES = 512 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d.get("hbm_gbs", 6650.0)), float(d.get("sm_max_mhz", 1965.0)), "measured"
    return 6650.0, 1965.0, "fallback"


# --------------------------------------------------------------------------
# algorithmic counts (one launch of each kernel), FP32 = 4 bytes
# --------------------------------------------------------------------------
def algorithmic(N, E, d_in, d_e, d_out, U, paths, coeff):
    """Bytes each kernel must move at least, and the forward/backward flops.

    forward : W, Y, col, rowptr, x (each once) in; out once
    backward: W, Y, col, rowptr, x, grad_out in; dW, dY out (the per-edge
              message buffer of the two-pass dx is an implementation choice and
              is not counted)
    bwd_reduce: the sender CSR in; dx out (the dY slice partials it also sums
              are part of the same implementation choice and not counted)
    sph_harm: r in; Y out
    flops (factored evaluation): forward per edge and path 2 nnz(C) for
      Chat = C . Y plus u (2 (2l1+1)(2l3+1) + 2 (2l3+1)); backward per edge and
      path 2 nnz + u (4 (2l1+1)(2l3+1) + 4 (2l3+1) + 2 nnz)
    """
    b = {
        "cgtp_fwd": 4 * (E * U + E * d_e + E + (N + 1) + N * d_in + N * d_out),
        "cgtp_bwd": 4 * (E * U + E * d_e + E + (N + 1) + N * d_in + N * d_out + E * U + E * d_e),
        "bwd_reduce": 4 * (N + 1 + E + N * d_in),
        "sph_harm": 4 * (3 * E + E * d_e),
    }
    ff = fb = 0.0
    for (l1, l2, l3, mul, xo, k0, oo, co) in paths:
        n1, n2, n3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
        nnz = int(np.count_nonzero(coeff[co:co + n1 * n2 * n3]))
        ff += 2 * nnz + mul * (2 * n1 * n3 + 2 * n3)
        fb += 2 * nnz + mul * (4 * n1 * n3 + 4 * n3 + 2 * nnz)
    return b, {"cgtp_fwd": ff * E, "cgtp_bwd": fb * E}


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception as e:  # nvidia-smi missing
            log("clock sampling unavailable:", e)
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [t.strip() for t in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        top = max(sm)
        loaded = [v for v in sm if v >= 0.5 * top] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# ranks: one process per GPU, independent replicas of the step
# --------------------------------------------------------------------------
def init_distributed(world: int, local_rank: int, backend: str = "nccl", timeout_s: int = 120) -> None:
    """Process group for N > 1 (RANK, WORLD_SIZE, MASTER_* from the launcher's
    environment).  The replicas exchange nothing on the data path: the group
    only brackets the timed region with barriers and takes the max time."""
    if world <= 1:
        return
    import datetime
    import torch
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time (a number of one rank for world == 1)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, units_per_rank: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank runs the full workload)."""
    return world * units_per_rank / (ms_max * 1e-3)


# --------------------------------------------------------------------------
# workload (host side)
# --------------------------------------------------------------------------
def build_workload(name: str, seed: int = 0):
    from equivariant_mlip_clebsch_b200 import cgtp as C
    c = WL.CONFIGS[name]
    plan = C.Plan(c["irreps_in"], c["irreps_edge"], c["irreps_out"], 6)
    pos, box = WL.si_diamond(c["cells"], c["sigma"], seed)
    rowptr, col, shift, r = C.neighbor_list(pos, box, c["rc"])
    N, E = len(pos), len(col)
    rpt, perm = C.csr_transpose(rowptr, col, N)
    muls = [int(t.split("x")[0]) for t in c["irreps_out"].split("+")]
    col_std = WL.column_std(muls, plan.out_fan_in())
    host = dict(rowptr=rowptr, col=col, rpt=rpt, perm=perm, r=r,
                x=WL.draw_x(N, plan.d_in, seed), W=WL.draw_W(E, plan.n_weights, col_std, seed),
                g=WL.draw_g(N, plan.d_out, seed))
    return plan, host, N, E, c


def workload_config(name: str, N: int, E: int, U: int, world: int) -> dict:
    """The ``config`` of both arms' JSON lines (identical dicts): the workload
    and what one step computes; how each arm times it is outside."""
    c = WL.CONFIGS[name]
    w_mb = 4.0 * E * U / 1e6
    return {"workload": f"{name}: {c['desc']}", "atoms": N, "edges": E,
            "irreps_in": c["irreps_in"], "irreps_edge": c["irreps_edge"], "irreps_out": c["irreps_out"],
            "seed": 0, "step": "sph_harm + forward + backward (dx, dW, dY)",
            "l2": (f"inputs larger than L2 (W alone {w_mb:.0f} MB)" if w_mb > 126 else
                   f"W is {w_mb:.0f} MB") + "; the GPU arm also writes a 512 MB buffer before every timed step",
            "parallelism": "replicas" if world > 1 else "single GPU"}


def fp32_peaks(dev, smax_mhz: float) -> dict:
    """FP32 peaks: derived (SMs from the device properties x 128 FP32 lanes x 2
    flop x the max SM clock) and measured (the library's FMA probe, best of
    three ~50 ms launches)."""
    import ctypes
    import torch
    from equivariant_mlip_clebsch_b200 import cgtp as C
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    derived = sms * 128 * 2 * smax_mhz * 1e6 / 1e12
    n = ctypes.c_int64()
    C._check(C._lib.cgtp_fma_peak_sink_floats(ctypes.byref(n)))
    sink = torch.empty(n.value, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    flops = ctypes.c_double()
    best = 0.0
    for iters in (2000, 100000, 100000, 100000):  # the first launch warms up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        C._check(C._lib.cgtp_fma_peak(iters, ctypes.c_void_p(sink.data_ptr()), n.value,
                                      ctypes.c_void_p(stream.cuda_stream), ctypes.byref(flops)))
        e1.record(stream)
        torch.cuda.synchronize()
        if iters > 2000:
            best = max(best, flops.value / (e0.elapsed_time(e1) * 1e-3) / 1e12)
    return {"derived_tflops": derived, "measured_tflops": best, "sms": sms, "sm_max_mhz": smax_mhz,
            "derived": f"{sms} SMs x 128 FP32 lanes x 2 flop x {smax_mhz:.0f} MHz",
            "measured": "cgtp_fma_peak: 2 CTAs x 512 threads per SM, 8 independent FMA chains, best of 3"}


def kernel_roofs(kt: dict, alg_b: dict, alg_f: dict, hbm: float, fp32: dict) -> dict:
    """Per kernel: average device time, achieved GB/s and TFLOP/s, the binding
    roof (HBM unless its flops at the derived FP32 peak take longer) and the
    fractions of HBM and of both FP32 peaks."""
    out = {}
    for nm, (ms, cnt) in kt.items():
        avg = ms / max(cnt, 1)
        d = {"avg_ms": avg, "launches": cnt}
        t = avg * 1e-3
        if nm in alg_b:
            d["GB/s"] = alg_b[nm] / t / 1e9
            d["frac_hbm"] = d["GB/s"] / hbm
        if nm in alg_f:
            d["TFLOP/s"] = alg_f[nm] / t / 1e12
            d["frac_fp32_derived"] = d["TFLOP/s"] / fp32["derived_tflops"]
            if fp32["measured_tflops"] > 0:
                d["frac_fp32_measured"] = d["TFLOP/s"] / fp32["measured_tflops"]
        if nm in alg_b and nm in alg_f:
            alu = alg_f[nm] / (fp32["derived_tflops"] * 1e12) > alg_b[nm] / (hbm * 1e9)
            d["bound"] = "alu" if alu else "hbm"
            d["frac_bound"] = d["frac_fp32_derived"] if alu else d["frac_hbm"]
        elif nm in alg_b:
            d["bound"] = "hbm"
            d["frac_bound"] = d["frac_hbm"]
        out[nm] = d
    return out


class Timer:
    """K timed repetitions of a callable on one stream, the L2 flushed before
    each (not timed); mean device milliseconds."""

    def __init__(self, flush, stream):
        self.flush, self.stream = flush, stream

    def __call__(self, fn, k: int) -> float:
        import torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for a, b in ev:
            self.flush.zero_()
            a.record(self.stream)
            fn()
            b.record(self.stream)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in ev]))


class Workbench:
    """One workload resident on the device, with its step, forward and the
    per-kernel breakdown."""

    def __init__(self, name, dev, flush):
        import torch
        t0 = time.time()
        self.name, self.dev = name, dev
        self.plan, self.host, self.N, self.E, self.c = build_workload(name)
        self.setup_s = time.time() - t0
        plan, N, E = self.plan, self.N, self.E
        self.T = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in self.host.items()}
        self.Y = torch.empty((E, plan.d_edge), device=dev)
        self.out = torch.empty((N, plan.d_out), device=dev)
        self.dx = torch.empty((N, plan.d_in), device=dev)
        self.dW = torch.empty((E, plan.n_weights), device=dev)
        self.dY = torch.empty((E, plan.d_edge), device=dev)
        self.ws = torch.empty(max(plan.workspace_size(N, N, E), 256), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream()
        self.timer = Timer(flush, self.stream)
        self.graph = None

    def step(self):
        T, plan = self.T, self.plan
        plan.sph_harm(T["r"], self.Y)
        plan.forward(T["rowptr"], T["col"], T["x"], self.Y, T["W"], out=self.out)
        plan.backward(T["rowptr"], T["col"], T["rpt"], T["perm"], T["x"], self.Y, T["W"], T["g"],
                      grads=(self.dx, self.dW, self.dY), workspace=self.ws)

    def fwd(self):
        T = self.T
        self.plan.sph_harm(T["r"], self.Y)
        self.plan.forward(T["rowptr"], T["col"], T["x"], self.Y, T["W"], out=self.out)

    def warm(self, n):
        import torch
        for _ in range(n):
            self.step()
        torch.cuda.synchronize()
        self.plan.check_device_error()

    def capture(self):
        import torch
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        self.graph.replay()
        torch.cuda.synchronize()
        self.plan.check_device_error()

    def measure(self, k: int, use_graph: bool):
        """(step ms, launched step ms, forward ms, kernel times {name: (ms, n)})."""
        if use_graph and self.graph is None:
            self.capture()
        ms_step = self.timer(self.graph.replay if use_graph else self.step, k)
        self.plan.kernel_times()  # discard
        self.plan.set_timing(True)
        ms_eager = self.timer(self.step, k)
        self.plan.set_timing(False)
        kt = self.plan.kernel_times()
        ms_fwd = self.timer(self.fwd, k)
        self.plan.check_device_error()
        return ms_step, ms_eager, ms_fwd, kt

    def algorithmic(self):
        p = self.plan
        return algorithmic(self.N, self.E, p.d_in, p.d_edge, p.d_out, p.n_weights, p.paths(), p.coefficients())

    def close(self):
        self.graph = None
        self.T = self.Y = self.out = self.dx = self.dW = self.dY = self.ws = None
        self.plan.close()


def per_workload_entry(wb: "Workbench", k: int, use_graph: bool, hbm: float, fp32: dict, world: int,
                       cpu_budget: float) -> dict:
    ms_step, ms_eager, ms_fwd, kt = wb.measure(k, use_graph)
    alg_b, alg_f = wb.algorithmic()
    N, E = wb.N, wb.E
    d = {"atoms": N, "edges": E, "steps": k,
         "fwd": {"ms": ms_fwd, "edges_per_s": world * E / (ms_fwd * 1e-3),
                 "atoms_per_s": world * N / (ms_fwd * 1e-3), "what": "sph_harm + forward"},
         "fwd_bwd": {"ms": ms_step, "edges_per_s": world * E / (ms_step * 1e-3),
                     "atoms_per_s": world * N / (ms_step * 1e-3),
                     "what": "sph_harm + forward + backward (dx, dW, dY)"
                             + (", replayed from one CUDA graph" if use_graph else "")},
         "ms_per_step_launched": ms_eager,
         "kernels": kernel_roofs(kt, alg_b, alg_f, hbm, fp32)}
    if cpu_budget > 0:
        try:
            s = oracle_sample(wb.name, cpu_budget)
            d["cpu_baseline"] = {"value": s["edges_per_s"], "unit": "edges/s",
                                 "atoms_per_s": s["edges_per_s"] * N / E, "cores": s["cores"],
                                 "kind": "oracle",
                                 "sample": f"receivers 0..{s['rows'] - 1} ({s['edges']} edges), harmonics + "
                                           f"forward + backward, {s['reps']} passes in {s['seconds']:.1f}s, FP64"}
        except Exception as e:  # reported; the GPU figures stand
            d["cpu_baseline"] = {"error": str(e)}
    return d


def sparse_field(wb: "Workbench", k: int, ms_dense_step: float, ms_dense_fwd: float) -> dict:
    """The BranchIP sparse evaluation (cgtp_sparse_forward / _backward, all
    four gradients) on the workload with 25, 50 and 75 % of the edges
    active, timed like the step (harmonics included, L2 flushed)."""
    import torch
    plan, T, E = wb.plan, wb.T, wb.E
    ws = torch.empty(max(plan.sparse_workspace_size(wb.N, wb.N, E), 256), dtype=torch.uint8, device=wb.dev)
    dg = torch.empty(E, device=wb.dev)
    out = {"what": "sph_harm + sparse forward (+ sparse backward: dx, dW, dY, dgate, zero-padded); gate "
                   "~ workloads.draw_gate (random edges, gate U(0,1] when active)"}
    for frac in (0.25, 0.5, 0.75):
        gate = torch.from_numpy(WL.draw_gate(E, frac)).to(wb.dev)
        n_act = int((gate > 0).sum().item())

        def fwd():
            plan.sph_harm(T["r"], wb.Y)
            plan.sparse_forward(T["rowptr"], T["col"], T["x"], wb.Y, T["W"], gate, out=wb.out, workspace=ws)

        def step():
            fwd()
            plan.sparse_backward(T["rowptr"], T["col"], T["rpt"], T["perm"], T["x"], wb.Y, T["W"], gate, T["g"],
                                 grads=(wb.dx, wb.dW, wb.dY, dg), workspace=ws)
        step()
        torch.cuda.synchronize()
        ms_f = wb.timer(fwd, k)
        ms_s = wb.timer(step, k)
        plan.check_device_error()
        out[f"{int(frac * 100)}%"] = {
            "active_edges": n_act, "fwd_ms": ms_f, "fwd_bwd_ms": ms_s,
            "fwd_bwd_edges_per_s": E / (ms_s * 1e-3), "active_edges_per_s": n_act / (ms_s * 1e-3),
            "speedup_vs_dense_fwd_bwd": ms_dense_step / ms_s, "speedup_vs_dense_fwd": ms_dense_fwd / ms_f}
    return out


def graph_check_cost(wb: "Workbench", k: int) -> dict:
    """Time of the device graph checks a checked call adds (the checks of
    the receiver CSR and of the sender lists, the read-back of their result
    and the wait for it), timed directly through cgtp_validate_graph."""
    T = wb.T

    def check():
        wb.plan.validate_graph(T["rowptr"], T["col"], wb.N, T["rpt"], T["perm"], stream=wb.stream)
    check()
    return {"ms_added": wb.timer(check, k), "what": "cgtp_validate_graph on the step's graph (receiver CSR "
            "and sender lists), host round trip included"}


def run_cgtp(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    name = args.config
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    wb = Workbench(name, dev, flush)
    plan, T, N, E, c = wb.plan, wb.T, wb.N, wb.E, wb.c
    log(f"[rank {rank}] plan + workload {name}: N={N} E={E} ({wb.setup_s:.1f}s)")
    stream = wb.stream
    wb.warm(args.warmup)
    if args.profile == "double_backward":  # for ncu: K double backwards (all three cotangents)
        gen = torch.Generator(device=dev).manual_seed(3)
        hx, hW, hY = (torch.randn(t.shape, device=dev, generator=gen) for t in (T["x"], T["W"], wb.Y))
        grads = tuple(torch.empty_like(t) for t in (T["g"], T["x"], T["W"], wb.Y))
        dws = torch.empty(max(plan.double_backward_workspace_size(N, N, E), 256), dtype=torch.uint8, device=dev)
        plan.prepare_double_backward()
        for _ in range(args.steps):
            flush.zero_()
            plan.double_backward(T["rowptr"], T["col"], T["rpt"], T["perm"], T["x"], wb.Y, T["W"], T["g"],
                                 h_x=hx, h_W=hW, h_Y=hY, grads=grads, workspace=dws)
        torch.cuda.synchronize()
        plan.check_device_error()
        return {"profile": name, "what": "double_backward", "steps": args.steps, "N": N, "E": E}
    if args.profile:  # for ncu: warm-up plus K plain steps, nothing else
        for _ in range(args.steps):
            flush.zero_()
            wb.step()
        torch.cuda.synchronize()
        plan.check_device_error()
        return {"profile": name, "steps": args.steps, "warmup": args.warmup, "N": N, "E": E}

    # keep the GPU busy ~1 s while the clock sampler warms up, then time K steps
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for _ in range(5):
            wb.step()
        torch.cuda.synchronize()
    use_graph = not args.no_graph
    if use_graph:
        wb.capture()
    # ---- the headline: K steps, barrier + synchronize on both sides
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_step_local = wb.timer(wb.graph.replay if use_graph else wb.step, args.steps)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_step = max_over_ranks(ms_step_local, world, dev)
    value = replica_value(world, E, ms_step)
    # ---- the per-kernel breakdown and the forward on the same workload
    _, ms_eager, fwd_ms, kt = wb.measure(args.steps, use_graph)

    # the force chain after the backward (dL/dY -> dL/dr -> forces), not in
    # the step: reported beside it
    from equivariant_mlip_clebsch_b200 import cgtp as C
    gr = torch.empty((E, 3), device=dev)
    Fo = torch.empty((N, 3), device=dev)

    def force_chain():
        plan.sph_harm_backward(T["r"], wb.dY, grad_r=gr)
        C.edge_forces(T["rowptr"], T["rpt"], T["perm"], gr, forces=Fo)
    force_ms = wb.timer(force_chain, args.steps)
    # the strain derivative (virial) from the same grad_r, timed on its own
    Vo = torch.empty((3, 3), device=dev)
    try:
        virial_ms = wb.timer(lambda: C.edge_virial(T["r"], gr, virial=Vo), args.steps)
        virial = {"ms": virial_ms, "edges_per_s": world * E / (virial_ms * 1e-3),
                  "achieved_gbs": 24.0 * E / (virial_ms * 1e-3) / 1e9,
                  "what": "edge_virial from grad_r (24 B/edge read), after the step (not in it)"}
    except (C.CgtpError, ValueError, TypeError) as e:  # reported, the headline stands
        virial = {"error": str(e)}
    # the double backward (all three cotangents), timed on its own
    try:
        gen = torch.Generator(device=dev).manual_seed(3)
        hx, hW, hY = (torch.randn(t.shape, device=dev, generator=gen) for t in (T["x"], T["W"], wb.Y))
        dgrads = tuple(torch.empty_like(t) for t in (T["g"], T["x"], T["W"], wb.Y))
        dws = torch.empty(max(plan.double_backward_workspace_size(N, N, E), 256), dtype=torch.uint8, device=dev)
        tangent = plan.prepare_double_backward()  # builds the tangent kernels outside the timing

        def dbl():
            plan.double_backward(T["rowptr"], T["col"], T["rpt"], T["perm"], T["x"], wb.Y, T["W"], T["g"],
                                 h_x=hx, h_W=hW, h_Y=hY, grads=dgrads, workspace=dws)
        dbl()
        torch.cuda.synchronize()
        dbl_ms = wb.timer(dbl, args.steps)
        plan.kernel_times()  # discard
        plan.set_timing(True)
        wb.timer(dbl, args.steps)
        plan.set_timing(False)
        dbl_kernels = {nm: {"avg_ms": ms / max(n, 1), "launches": n} for nm, (ms, n) in plan.kernel_times().items()}
        # the operation's own bytes: x, Y, W, grad_out and the three cotangents
        # read once, the four gradients written once, both CSRs read
        dbl_bytes = 4 * (2 * N * plan.d_in + 2 * E * plan.d_edge + 2 * E * plan.n_weights + N * plan.d_out
                         + N * plan.d_out + N * plan.d_in + E * plan.n_weights + E * plan.d_edge
                         + 2 * (N + 1 + E))
        double_backward = {"ms": dbl_ms, "edges_per_s": world * E / (dbl_ms * 1e-3),
                           "algorithmic_bytes": dbl_bytes, "achieved_gbs": dbl_bytes / (dbl_ms * 1e-3) / 1e9,
                           "vs_step": dbl_ms / ms_step_local,
                           "path": ("tangent backward + one plain and two accumulating forwards"
                                    if "double backward forward=sum" in plan.describe() else
                                    "tangent kernels (one forward, one backward pass)") if tangent else
                                   "composition of forwards and backwards",
                           "what": "double_backward with h_x, h_W, h_Y, after the step (not in it)",
                           "kernels": dbl_kernels}
        del hx, hW, hY, dgrads, dws
    except (C.CgtpError, ValueError, TypeError) as e:  # reported, the headline stands
        double_backward = {"error": str(e)}
    # BranchIP sparse evaluation at 25 / 50 / 75 % active edges, after the step
    try:
        sparse = sparse_field(wb, args.steps, ms_step_local, fwd_ms)
    except (C.CgtpError, ValueError, TypeError) as e:  # reported, the headline stands
        sparse = {"error": str(e)}
    hbm, smax, pk_kind = peaks()
    if "achieved_gbs" in double_backward:
        double_backward["frac_hbm"] = double_backward["achieved_gbs"] / hbm
    fp32 = fp32_peaks(dev, smax)
    clocks_main = sampler.stop()
    plan.check_device_error()

    # ---- roofline of the dominant kernel
    alg_b, alg_f = wb.algorithmic()
    kernels = kernel_roofs(kt, alg_b, alg_f, hbm, fp32)
    timed_names = [n for n in kt if n in ("cgtp_fwd", "cgtp_bwd")]
    dom = max(timed_names, key=lambda n: kt[n][0]) if timed_names else max(kt, key=lambda n: kt[n][0])
    kd = kernels[dom]
    if kd.get("bound") == "alu":
        roof = {"bound": "alu", "achieved": kd["TFLOP/s"], "peak": fp32["derived_tflops"], "unit": "TFLOP/s",
                "peak_source": fp32["derived"], "measured_fma_peak": fp32["measured_tflops"],
                "frac_of_measured_fma_peak": kd.get("frac_fp32_measured")}
    else:
        roof = {"bound": "hbm", "achieved": kd["GB/s"], "peak": hbm, "unit": "GB/s",
                "peak_source": pk_kind + " (MEASURED_PEAKS.json hbm_gbs)",
                "frac_vs_spec_8000": kd["GB/s"] / 8000.0}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["kernel_hashes"] = kernel_hashes(plan)
    roof["algorithmic_bytes_per_launch"] = alg_b.get(dom)
    roof["traffic"] = ncu_traffic(name, dom, plan)
    roof["fp32_sgemm_tflops"] = sgemm_tflops(dev)  # measured cuBLAS FP32 (CUDA cores), context
    gpu_launches = sum(cnt for nm, (ms, cnt) in kt.items() if nm != "zero_fill")

    # ---- end to end through the same API with host buffers
    e2e = run_e2e(args, plan, T, wb.host, wb.Y, wb.out, wb.dx, wb.dW, wb.dY, wb.ws, E, dev, world)
    res = dict(metric=METRIC, value=value, unit="edges/s", n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="f32", data="synthetic",
               config=workload_config(name, N, E, plan.n_weights, world),
               timing={"device": "CUDA events on the launching stream, K steps"
                                 + (" replayed from one CUDA graph" if use_graph else " launched call by call"),
                       "l2_flush": f"{L2_FLUSH_BYTES >> 20} MB buffer written before every timed step (not timed)"},
               atoms_per_s=replica_value(world, N, ms_step),
               fwd_edges_per_s=world * E / (fwd_ms * 1e-3), fwd_atoms_per_s=world * N / (fwd_ms * 1e-3),
               fwd_ms=fwd_ms, ms_per_step_launched=ms_eager,
               force_chain={"ms": force_ms, "edges_per_s": world * E / (force_ms * 1e-3),
                            "what": "sph_harm_backward + edge_forces after the step (not in it)"},
               virial=virial, double_backward=double_backward, sparse=sparse,
               roofline=roof, fp32_peak=fp32, kernels=kernels, gpu_launches=int(gpu_launches), e2e=e2e,
               clocks=clocks_main)
    # the five workloads of the target and Table 1 Cases 4-6, each measured on
    # its own (the headline workload's figures are taken again in the same
    # way, for one table)
    if not args.no_per_workload:
        per = {}
        k = max(3, min(args.steps, 10))
        wb.close()
        del wb
        torch.cuda.empty_cache()
        sampler2 = ClockSampler(sampler.idx)
        sampler2.start()
        for nm in PER_WORKLOAD:
            try:
                w2 = Workbench(nm, dev, flush)
                w2.warm(3)
                per[nm] = per_workload_entry(w2, k, use_graph, hbm, fp32, world,
                                             args.cpu_budget / 4 if rank == 0 else 0.0)
                per[nm]["graph_checks"] = graph_check_cost(w2, k)
                per[nm]["plan_and_graph_s"] = w2.setup_s
                w2.close()
                del w2
                torch.cuda.empty_cache()
            except Exception as e:  # reported, the headline stands
                per[nm] = {"error": f"{type(e).__name__}: {e}"}
            log(f"[rank {rank}] per-workload {nm}: "
                + (f"{per[nm]['fwd_bwd']['edges_per_s']:.3e} edges/s" if "fwd_bwd" in per[nm] else per[nm]["error"]))
        per["clocks"] = sampler2.stop()
        res["per_workload"] = per
    return res


def sgemm_tflops(dev) -> float:
    """FP32 throughput of CUDA-core work as measured here: a cuBLAS FP32 GEMM
    (TF32 off), 8192^3, best of three.  Reported beside the derived FP32 peak."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        n = 8192
        a = torch.randn(n, n, device=dev)
        b = torch.randn(n, n, device=dev)
        c = torch.empty(n, n, device=dev)
        torch.matmul(a, b, out=c)
        torch.cuda.synchronize()
        best = 1e30
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def run_e2e(args, plan, T, host, Y, out, dx, dW, dY, ws, E, dev, world):
    """The step through the public API with host buffers: every step copies its
    inputs (r, x, W, g) from pinned host memory and reads its results (out,
    dx, dW, dY) back.  Steps are pipelined over three streams (host->device,
    compute, device->host) and two buffer sets, so one step's read-back
    overlaps the next step's upload on the full-duplex link; ordering by
    events.  Time = first upload to last read-back, CUDA events."""
    import torch
    names = ("r", "x", "W", "g")
    pin = {k: torch.from_numpy(np.ascontiguousarray(host[k])).pin_memory() for k in names}
    dsts = [{k: torch.empty_like(T[k]) for k in names} for _ in range(2)]
    outs = [[out, dx, dW, dY], [torch.empty_like(t) for t in (out, dx, dW, dY)]]
    Ys = [Y, torch.empty_like(Y)]
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs[0]]
    s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    steps = max(3, min(args.steps, 20))
    ev = lambda: torch.cuda.Event()

    def run(n, a=None, b=None):
        computed = [None, None]  # compute of the set's last step done (inputs free)
        drained = [None, None]   # read-back of the set's last step done (outputs free)
        if a is not None:
            a.record(s_in)
        for k in range(n):
            q = k & 1
            d, o = dsts[q], outs[q]
            if computed[q] is not None:
                s_in.wait_event(computed[q])
            for nm in names:
                with torch.cuda.stream(s_in):
                    d[nm].copy_(pin[nm], non_blocking=True)
            up = ev()
            up.record(s_in)
            s_c.wait_event(up)
            if drained[q] is not None:
                s_c.wait_event(drained[q])
            plan.sph_harm(d["r"], Ys[q], stream=s_c)
            plan.forward(T["rowptr"], T["col"], d["x"], Ys[q], d["W"], out=o[0], stream=s_c)
            plan.backward(T["rowptr"], T["col"], T["rpt"], T["perm"], d["x"], Ys[q], d["W"], d["g"],
                          grads=(o[1], o[2], o[3]), workspace=ws, stream=s_c)
            done = ev()
            done.record(s_c)
            computed[q] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                for h, t in zip(hout, o):
                    h.copy_(t, non_blocking=True)
            dr = ev()
            dr.record(s_out)
            drained[q] = dr
        if b is not None:
            b.record(s_out)

    run(2)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, a, b)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return {"value": replica_value(world, E, ms), "unit": "edges/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps,
            "pipelined": "host->device, compute and device->host on three streams, two buffer sets"}


def kernel_hashes(plan) -> dict:
    """The generated kernels' source hashes (as compiled in this process),
    which key the committed ncu traffic figures."""
    out = {}
    for line in plan.describe().splitlines():
        for tag, key in (("forward:", "cgtp_fwd"), ("backward:", "cgtp_bwd"), ("backward (edge ranges", "cgtp_bwd_er")):
            if line.startswith(tag) and "hash=" in line:
                out[key] = line.split("hash=")[1].split()[0]
    return out


def ncu_traffic(name, kernel, plan):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the same generated kernel (matching source hash); else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(f"{name}/{kernel}")
    except Exception:
        return None
    if not d:
        return None
    desc = plan.describe()
    tag = "forward" if kernel == "cgtp_fwd" else "backward"
    for line in desc.splitlines():  # either backward variant
        if line.startswith(tag) and f"hash={d.get('kernel_hash')}" in line:
            return d.get("bytes_per_launch")
    return None


# --------------------------------------------------------------------------
# the oracle on the host cores: cpu_baseline and the reference arm
# --------------------------------------------------------------------------
def oracle_sample(name: str, budget_s: float, rows: int | None = None, nthreads: int = 0,
                  backward: bool = True):
    """Time the FP64 oracle (forward + backward, all three gradients; the
    forward alone with backward=False) on the sub-graph of the first ``rows``
    receivers, repeated until ``budget_s``; nthreads 0 = all host cores."""
    import oracle as O
    c = WL.CONFIGS[name]
    pos, box = WL.si_diamond(c["cells"], c["sigma"], 0)
    rowptr, col, shift, vec = O.neighbor_list(pos, box, c["rc"])
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    N = len(pos)
    fan = np.zeros(len(P.irreps_out), dtype=int)
    bases = np.concatenate([[0], np.cumsum([m for m, _, _ in P.irreps_out])])
    for k0 in P.table[:, 5]:
        fan[np.searchsorted(bases, k0, side="right") - 1] += 1
    std = WL.column_std([m for m, _, _ in P.irreps_out], fan)
    if rows is None:
        # size the sample from a quick probe so one pass costs ~budget/3
        rows = min(N, 32)
        rp = rowptr[:rows + 1]
        t = time.time()
        _oracle_pass(O, P, rp, col, vec, N, std, pos, nthreads, backward)
        dt = max(time.time() - t, 1e-3)
        rows = int(min(N, max(8, rows * (budget_s / 3) / dt)))
    rp = rowptr[:rows + 1]
    nE = int(rp[-1])
    reps, t0 = 0, time.time()
    while True:
        _oracle_pass(O, P, rp, col, vec, N, std, pos, nthreads, backward)
        reps += 1
        if time.time() - t0 >= budget_s or reps >= 50:
            break
    dt = time.time() - t0
    return {"edges_per_s": reps * nE / dt, "rows": rows, "edges": nE, "reps": reps, "seconds": dt,
            "cores": nthreads or O.max_threads()}


def _oracle_pass(O, P, rp, col, vec, N, std, pos, nthreads=0, backward=True):
    E = int(rp[-1])
    x = WL.draw_x(N, P.D_in)
    W = WL.draw_W(E, P.U, std)
    g = WL.draw_g(len(rp) - 1, P.D_out)
    Y = O.sph_harm(P.L, vec[:E].astype(np.float32))
    O.forward(P, rp, col[:E], x, Y, W, nthreads=nthreads)
    if backward:
        O.backward(P, rp, col[:E], N, x, Y, W, g, nthreads=nthreads)


def run_reference(args, rank, world):
    if rank != 0:
        return None
    name = args.config
    c = WL.CONFIGS[name]
    per = max(2.0, min(20.0, 120.0 / max(args.steps + args.warmup, 1)))
    s = oracle_sample(name, per)
    rows = s["rows"]
    times = []
    import oracle as O
    pos, box = WL.si_diamond(c["cells"], c["sigma"], 0)
    rowptr, col, shift, vec = O.neighbor_list(pos, box, c["rc"])
    P = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"])
    std = np.ones(P.U)
    rp = rowptr[:rows + 1]
    for k in range(args.warmup + args.steps):
        t = time.time()
        _oracle_pass(O, P, rp, col, vec, len(pos), std, pos)
        if k >= args.warmup:
            times.append(time.time() - t)
    nE = int(rp[-1])
    value = nE / float(np.mean(times))
    sample = (f"receivers 0..{rows - 1} of {len(pos)} ({nE} of {len(col)} edges), harmonics + "
              f"forward + backward per step, FP64")
    return dict(impl="reference", metric=METRIC, value=value, unit="edges/s", n_gpus=world,
                steps=args.steps, warmup=args.warmup, ms_per_step=float(np.mean(times)) * 1e3,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=workload_config(name, len(pos), int(len(col)), P.U, world),
                timing={"host": "wall clock per step of the FP64 oracle on the host cores, on a bounded "
                                "sample of the workload's receivers"},
                cpu_baseline={"value": value, "unit": "edges/s", "cores": s["cores"], "kind": "oracle",
                              "sample": sample},
                e2e={"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cgtp", choices=["cgtp", "reference"])
    ap.add_argument("--no-graph", action="store_true",
                    help="time the step launched kernel by kernel instead of from a CUDA graph")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(WL.CONFIGS))
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline field (0 to skip)")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-workload figures of the five workloads")
    ap.add_argument("--profile", nargs="?", const="step", default=None, choices=["step", "double_backward"],
                    help="warm-up + K steps only (no clock loop, e2e or CPU baseline), for ncu; "
                         "'double_backward': K double backwards with all three cotangents instead")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    init_distributed(world, local_rank, "nccl")
    res = run_cgtp(args, rank, world, local_rank)
    if rank == 0 and args.cpu_budget > 0 and not args.profile:
        s = oracle_sample(args.config, args.cpu_budget)
        res["cpu_baseline"] = {"value": s["edges_per_s"], "unit": "edges/s", "cores": s["cores"],
                               "kind": "oracle",
                               "sample": f"receivers 0..{s['rows'] - 1} ({s['edges']} edges), harmonics + "
                                         f"forward + backward, {s['reps']} passes in {s['seconds']:.1f}s, FP64"}
        # the same step on one host thread, and the forward alone on all cores
        for key, kw in (("single_thread", dict(nthreads=1)), ("forward_only", dict(backward=False))):
            v = oracle_sample(args.config, args.cpu_budget / 4, **kw)
            res["cpu_baseline"][key] = {"value": v["edges_per_s"], "unit": "edges/s", "cores": v["cores"],
                                        "sample": f"receivers 0..{v['rows'] - 1} ({v['edges']} edges), "
                                                  f"{v['reps']} passes in {v['seconds']:.1f}s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
