#!/usr/bin/env python
"""CGTP convolution throughput on B200.

One step = the whole hot path over one synthetic workload: real spherical
harmonics of the edge vectors, the forward CGTP convolution and its backward
(dL/dx, dL/dW, dL/dY).  The plan (paths, CG tables, kernel compilation) is
built once before timing.  Inputs are resident in HBM for ``value``; ``e2e``
repeats the step through the same public API with the inputs copied from
pinned host memory and the outputs copied back inside the timed region.

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
DEFAULT_CONFIG = "lmax2"  # the Lmax=2 channelwise workload the metric is quoted on
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


def run_cgtp(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    name = args.config
    t0 = time.time()
    plan, host, N, E, c = build_workload(name)
    log(f"[rank {rank}] plan + workload {name}: N={N} E={E} ({time.time() - t0:.1f}s)")
    T = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in host.items()}
    Y = torch.empty((E, plan.d_edge), device=dev)
    out = torch.empty((N, plan.d_out), device=dev)
    dx = torch.empty((N, plan.d_in), device=dev)
    dW = torch.empty((E, plan.n_weights), device=dev)
    dY = torch.empty((E, plan.d_edge), device=dev)
    ws = torch.empty(max(plan.workspace_size(N, N, E), 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(r_, x_, W_, g_):
        plan.sph_harm(r_, Y)
        plan.forward(T["rowptr"], T["col"], x_, Y, W_, out=out)
        plan.backward(T["rowptr"], T["col"], T["rpt"], T["perm"], x_, Y, W_, g_, grads=(dx, dW, dY),
                      workspace=ws)

    for _ in range(args.warmup):
        step(T["r"], T["x"], T["W"], T["g"])
    torch.cuda.synchronize()
    plan.check_device_error()
    if args.profile:  # for ncu: warm-up plus K plain steps, nothing else
        for _ in range(args.steps):
            flush.zero_()
            step(T["r"], T["x"], T["W"], T["g"])
        torch.cuda.synchronize()
        plan.check_device_error()
        return {"profile": name, "steps": args.steps, "warmup": args.warmup, "N": N, "E": E}

    # keep the GPU busy ~1 s while the clock sampler warms up, then time K steps
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for _ in range(20):
            step(T["r"], T["x"], T["W"], T["g"])
        torch.cuda.synchronize()
    # the step's four launches captured once in a CUDA graph (no launch gaps);
    # the headline times K replays
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(T["r"], T["x"], T["W"], T["g"])
        graph.replay()
        torch.cuda.synchronize()
        plan.check_device_error()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    ev_e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    ev_f = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()  # L2 flush (not timed)
        a, b = ev[k]
        a.record(stream)
        if graph is not None:
            graph.replay()
        else:
            step(T["r"], T["x"], T["W"], T["g"])
        b.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # the same K steps launched one by one, with the library's per-kernel
    # events on: the per-kernel breakdown and the roofline
    plan.kernel_times()  # discard
    plan.set_timing(True)
    for k in range(args.steps):
        flush.zero_()
        a, b = ev_e[k]
        a.record(stream)
        step(T["r"], T["x"], T["W"], T["g"])
        b.record(stream)
    torch.cuda.synchronize()
    plan.set_timing(False)
    kt = plan.kernel_times()  # the kernels of the K eager steps
    ms_eager = float(np.mean([a.elapsed_time(b) for a, b in ev_e]))
    # forward-only steps (harmonics + forward), for the forward edges/s
    for k in range(args.steps):
        flush.zero_()
        a, b = ev_f[k]
        a.record(stream)
        plan.sph_harm(T["r"], Y)
        plan.forward(T["rowptr"], T["col"], T["x"], Y, T["W"], out=out)
        b.record(stream)
    # the force chain after the backward (dL/dY -> dL/dr -> forces), not in
    # the step: reported beside it
    from equivariant_mlip_clebsch_b200 import cgtp as C
    gr = torch.empty((E, 3), device=dev)
    Fo = torch.empty((N, 3), device=dev)
    ev_c = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()
        a, b = ev_c[k]
        a.record(stream)
        plan.sph_harm_backward(T["r"], dY, grad_r=gr)
        C.edge_forces(T["rowptr"], T["rpt"], T["perm"], gr, forces=Fo)
        b.record(stream)
    # the strain derivative (virial) from the same grad_r, timed on its own
    Vo = torch.empty((3, 3), device=dev)
    ev_v = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    virial_err = None
    try:
        for k in range(args.steps):
            flush.zero_()
            a, b = ev_v[k]
            a.record(stream)
            C.edge_virial(T["r"], gr, virial=Vo)
            b.record(stream)
    except (C.CgtpError, ValueError, TypeError) as e:  # reported, the headline stands
        virial_err = str(e)
    # the double backward (all three cotangents), timed on its own
    ev_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    dbl_err = None
    try:
        gen = torch.Generator(device=dev).manual_seed(3)
        hx, hW, hY = (torch.randn(t.shape, device=dev, generator=gen) for t in (T["x"], T["W"], Y))
        dgrads = tuple(torch.empty_like(t) for t in (T["g"], T["x"], T["W"], Y))
        dws = torch.empty(max(plan.double_backward_workspace_size(N, N, E), 256), dtype=torch.uint8, device=dev)
        for k in range(args.steps):
            flush.zero_()
            a, b = ev_d[k]
            a.record(stream)
            plan.double_backward(T["rowptr"], T["col"], T["rpt"], T["perm"], T["x"], Y, T["W"], T["g"],
                                 h_x=hx, h_W=hW, h_Y=hY, grads=dgrads, workspace=dws)
            b.record(stream)
    except (C.CgtpError, ValueError, TypeError) as e:  # reported, the headline stands
        dbl_err = str(e)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    plan.check_device_error()
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    ms_fwd = [a.elapsed_time(b) for a, b in ev_f]
    force_ms = float(np.mean([a.elapsed_time(b) for a, b in ev_c]))
    if virial_err is None:
        virial_ms = float(np.mean([a.elapsed_time(b) for a, b in ev_v]))
        virial = {"ms": virial_ms, "edges_per_s": world * E / (virial_ms * 1e-3),
                  "achieved_gbs": 24.0 * E / (virial_ms * 1e-3) / 1e9,
                  "what": "edge_virial from grad_r (24 B/edge read), after the step (not in it)"}
    else:
        virial = {"error": virial_err}
    if dbl_err is None:
        dbl_ms = float(np.mean([a.elapsed_time(b) for a, b in ev_d]))
        # the operation's own bytes: x, Y, W, grad_out and the three cotangents
        # read once, the four gradients written once, both CSRs read
        dbl_bytes = 4 * (2 * N * plan.d_in + 2 * E * plan.d_edge + 2 * E * plan.n_weights + N * plan.d_out
                         + N * plan.d_out + N * plan.d_in + E * plan.n_weights + E * plan.d_edge
                         + 2 * (N + 1 + E))
        double_backward = {"ms": dbl_ms, "edges_per_s": world * E / (dbl_ms * 1e-3),
                           "algorithmic_bytes": dbl_bytes, "achieved_gbs": dbl_bytes / (dbl_ms * 1e-3) / 1e9,
                           "what": "double_backward with h_x, h_W, h_Y (3 forwards, 3 backwards, adds), "
                                   "after the step (not in it); achieved_gbs counts the operation's own "
                                   "bytes, so the composition's extra passes show as a low fraction"}
    else:
        double_backward = {"error": dbl_err}
    ms_step = max_over_ranks(float(np.sum(ms_steps)) / args.steps, world, dev)
    value = replica_value(world, E, ms_step)
    fwd_ms = float(np.mean(ms_fwd))

    # ---- per-kernel roofline (device time from the library's events)
    hbm, smax, pk_kind = peaks()
    if "achieved_gbs" in double_backward:
        double_backward["frac_hbm"] = double_backward["achieved_gbs"] / hbm
    paths = plan.paths()
    coeff = plan.coefficients()
    alg_b, alg_f = algorithmic(N, E, plan.d_in, plan.d_edge, plan.d_out, plan.n_weights, paths, coeff)
    kernels = {}
    for nm, (ms, cnt) in kt.items():
        avg = ms / max(cnt, 1)
        d = {"avg_ms": avg, "launches": cnt}
        if nm in alg_b:
            d["GB/s"] = alg_b[nm] / (avg * 1e-3) / 1e9
        if nm in alg_f:
            d["TFLOP/s"] = alg_f[nm] / (avg * 1e-3) / 1e12
        kernels[nm] = d
    timed_names = [n for n in kt if n in ("cgtp_fwd", "cgtp_bwd")]
    dom = max(timed_names, key=lambda n: kt[n][0]) if timed_names else max(kt, key=lambda n: kt[n][0])
    fp32_peak = 148 * 128 * 2 * smax * 1e6 / 1e12  # TFLOP/s at the max SM clock
    avg_dom = kt[dom][0] / kt[dom][1]
    bytes_dom = alg_b.get(dom, 0)
    flops_dom = alg_f.get(dom, 0.0)
    t_hbm = bytes_dom / (hbm * 1e9)
    t_alu = flops_dom / (fp32_peak * 1e12)
    if t_alu > t_hbm:
        roof = {"bound": "alu", "achieved": flops_dom / (avg_dom * 1e-3) / 1e12, "peak": fp32_peak,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": bytes_dom / (avg_dom * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "hbm":  # against the ~8 TB/s spec as well
        roof["frac_vs_spec_8000"] = roof["achieved"] / 8000.0
    roof["fp32_sgemm_tflops"] = sgemm_tflops(dev)  # measured FP32 (CUDA cores), context
    roof["kernel"] = dom
    roof["peak_source"] = pk_kind if roof["bound"] == "hbm" else \
        "148 SMs x 128 FP32 lanes x 2 flop x max SM clock"
    roof["traffic"] = ncu_traffic(name, dom, plan)
    gpu_launches = sum(cnt for nm, (ms, cnt) in kt.items() if nm != "zero_fill")

    # ---- end to end through the same API with host buffers
    e2e = run_e2e(args, plan, T, host, Y, out, dx, dW, dY, ws, E, dev, world)
    res = dict(metric=METRIC, value=value, unit="edges/s", n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="f32", data="synthetic",
               config={"workload": f"{name}: {c['desc']}", "atoms": N, "edges": E,
                       "irreps_in": c["irreps_in"], "irreps_edge": c["irreps_edge"],
                       "irreps_out": c["irreps_out"], "seed": 0,
                       "step": "sph_harm + forward + backward (dx, dW, dY)"
                               + (", replayed from one CUDA graph" if graph is not None else ""),
                       "l2": f"{L2_FLUSH_BYTES >> 20} MB buffer written before every timed step (not timed)",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
               atoms_per_s=replica_value(world, N, ms_step),
               fwd_edges_per_s=world * E / (fwd_ms * 1e-3), fwd_ms=fwd_ms,
               ms_per_step_launched=ms_eager,
               force_chain={"ms": force_ms, "edges_per_s": world * E / (force_ms * 1e-3),
                            "what": "sph_harm_backward + edge_forces after the step (not in it)"},
               virial=virial, double_backward=double_backward,
               roofline=roof, kernels=kernels, gpu_launches=int(gpu_launches), e2e=e2e, clocks=clocks)
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
                config={"workload": f"{name}: {c['desc']}", "atoms": len(pos), "edges": int(len(col))},
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
    ap.add_argument("--profile", action="store_true",
                    help="warm-up + K steps only (no clock loop, e2e or CPU baseline), for ncu")
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
