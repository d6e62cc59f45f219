"""The multi-replica bookkeeping of bench.py on CPU: two gloo ranks.

Each rank is an independent replica (the path shards by sequence and needs no
collective); the whole-job time is the slowest rank's and the value sums the
tokens of all ranks.  Runs two processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        elapsed = [0.5, 2.0][rank]               # rank 1 is the slow one
        t, v = bench.combine_ranks(elapsed, tokens_per_rank=1000.0, world=world, device="cpu")
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_sum_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, v in res:
        assert t == 2.0
        assert v == pytest.approx(2 * 1000.0 / 2.0)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    t, v = bench.combine_ranks(0.25, 100.0, 1)
    assert t == 0.25 and v == pytest.approx(400.0)


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched the driver's way for N = 2: rank 0 alone
    runs the oracle and prints one JSON line; the other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "0", "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"
