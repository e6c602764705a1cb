"""The N > 1 launch path on CPU: two ranks with the gloo backend.

bench.py runs one process per GPU, each on its own batch of the workload (weak
scaling, no collective on the data path); the only cross-rank step is the max of
the timed durations and the barriers around the timed loop.  These tests run that
plumbing as two real processes on the host, and launch the reference arm under
torchrun with two ranks: rank 0 alone prints its line, the other exits cleanly."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    ranks = bench.Ranks(world, rank, "gloo", torch.device("cpu"), timeout_s=60)
    ranks.barrier()
    per_rank_ms = [12.5, 20.0][rank]        # this rank's timed total
    mx = ranks.max(per_rank_ms)
    ranks.barrier()
    ranks.close()
    out_q.put((rank, mx, bench.weak_scaling_rate(world, 10, 16384, mx)))


def test_two_rank_max_and_weak_scaling_rate_over_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, rate in res:
        assert mx == 20.0                               # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 10 * 16384 / 0.020)  # units of all ranks / max time


def test_world_one_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    r = bench.Ranks(1, 0, "gloo", torch.device("cpu"))
    r.barrier()
    assert r.max(3.5) == 3.5
    r.close()


def test_reference_arm_under_torchrun_two_ranks():
    """bench.py --impl reference, launched as the scaling run launches it: rank 0 prints
    one JSON line with n_gpus = 2, rank 1 prints nothing and exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny_fp32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
