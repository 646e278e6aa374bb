"""Host-side logic of several ranks, on the CPU with the gloo backend.

bench.py runs one replica per GPU (the path shards into independent images; no
data-path collective).  What crosses ranks is a barrier and the maximum of the
timings, and the whole-job rate is the units of all replicas over the slowest
rank's time.  These tests run that logic in two gloo processes, and the reference
arm (the CPU oracle) under torchrun with two ranks, where rank 0 alone prints.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports times (r + 1, 5 - r, 2.5): the maximum over ranks is (2, 5, 2.5)
        got = bench.max_over_ranks([rank + 1.0, 5.0 - rank, 2.5], world)
        rate = bench.replica_rate(1000, world, got[0])
        q.put((rank, got, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_rate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, got, rate in res:
        assert got == [2.0, 5.0, 2.5]
        # 2 replicas x 1000 units in 2 ms (the slower rank's time)
        assert rate == pytest.approx(2 * 1000 / 2e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5], 1) == [3.0, 4.5]
    assert bench.replica_rate(10, 1, 0.0) == 0.0


def test_reference_arm_under_torchrun_two_ranks():
    """The reference arm is launched like the product arm; rank 0 alone runs the
    oracle and prints one JSON line, the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--config", "vit14_fp32", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
