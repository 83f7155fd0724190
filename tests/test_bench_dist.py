"""The N > 1 path of bench.py on the CPU: two ranks over gloo (127.0.0.1).

Replicas exchange nothing on the data path; the process group brackets the
timed region and takes the slowest rank's time, and rank 0 reports the
whole-job throughput (units of all ranks over that time).  These tests run the
same helpers bench.py uses, with the gloo backend instead of NCCL.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        bench.init_distributed(world, rank, backend="gloo", timeout_s=30)
        dist.barrier()  # as around the timed region
        ms = bench.max_over_ranks(1.0 + 2.0 * rank, world)  # ranks took 1 ms and 3 ms
        value = bench.replica_value(world, 21504, ms)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, ms, value, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, None, None, repr(e)))


def _run(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    try:
        for _ in range(world):
            out.append(q.get(timeout=90))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return sorted(out)


def test_two_ranks_take_the_slowest_time():
    res = _run(2)
    for rank, ms, value, err in res:
        assert err is None, err
        assert ms == pytest.approx(3.0)
        # both ranks processed 21504 edges; the job's time is the slower rank's
        assert value == pytest.approx(2 * 21504 / 3e-3)


def test_single_rank_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.init_distributed(1, 0)  # no process group for one rank
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.replica_value(1, 1000, 2.0) == pytest.approx(5e5)


def test_reference_arm_under_torchrun_prints_one_line():
    """bench.py --impl reference with two ranks: rank 0 times the oracle and
    prints one JSON line; rank 1 exits 0 without work."""
    import json
    import subprocess

    import bench
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    # the same metric, unit, direction and workload as the CUDA arm
    assert d["metric"] == bench.METRIC and d["unit"] == "edges/s" and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith(bench.DEFAULT_CONFIG + ":")
    # the config dict is the one the CUDA arm prints for the same workload
    import oracle as O
    from equivariant_mlip_clebsch_b200 import workloads as WL
    c = WL.CONFIGS[bench.DEFAULT_CONFIG]
    U = O.enumerate_paths(c["irreps_in"], c["irreps_edge"], c["irreps_out"]).U
    assert d["config"] == bench.workload_config(bench.DEFAULT_CONFIG, d["config"]["atoms"],
                                                d["config"]["edges"], U, 2)
    assert d["steps"] == 1 and d["warmup"] == 3 and d["cpu_baseline"]["cores"] >= 1
