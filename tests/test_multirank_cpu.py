"""The N > 1 bench path's host logic on two gloo ranks (CPU, no GPU): every
rank runs its own prompt, and the job's figures are the slowest rank's step
time and the sum of all ranks' FLOPs."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, q):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: step time 10 + r ms, 1e12 * (r + 1) FLOPs
        ms, flops, value = bench.aggregate(10.0 + rank, 1e12 * (rank + 1), ws)
        q.put((rank, ms, flops, value))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregate_two_ranks():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(ws))
    for rank, ms, flops, value in got:
        assert ms == pytest.approx(11.0)          # the slowest rank
        assert flops == pytest.approx(3e12)       # all ranks' work
        assert value == pytest.approx(3e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.aggregate(5.0, 2e12, 1) == (5.0, 2e12, pytest.approx(400.0))


def test_reference_arm_under_torchrun_prints_once():
    # launched like the scaling run (torchrun, two ranks on this host): rank 0
    # alone runs the oracle and prints one JSON line; the other rank exits 0
    # without work
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--seq-len", "4096", "--ref-total-budget", "2"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
