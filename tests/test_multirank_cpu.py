"""Multi-rank host logic on the CPU (gloo, world size 2).

The decode has no cross-sequence exchange, so N GPUs run N independent
replicas: the only collective steps are the barriers around the timed region
and the maximum of the device times over ranks.  These tests run that logic
with the gloo backend in separate processes, and the reference arm under
torchrun (rank 0 prints the one JSON line, the other ranks exit without work).
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        ms = bench.max_over_ranks(1.5 + rank, ws)           # rank r took 1.5 + r ms per step
        ph = [bench.max_over_ranks(10.0 * (r + 1) * (1 + rank), ws) for r in range(3)]
        v = bench.job_tokens_per_s(16, ws, ms)
        bench.barrier(ws)
        q.put((rank, ms, ph, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, ms, ph, v in got:
        assert ms == 2.5                                     # the slower rank's time
        assert ph == [20.0, 40.0, 60.0]
        assert v == pytest.approx(16 * 2 / 2.5e-3)           # all ranks' sequences over the slowest step


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-ctx", "32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
