"""Host-side multi-rank logic of bench.py on CPU with the gloo backend
(world size 2): max-over-ranks timing, whole-job weak-scaling throughput,
per-rank workloads, and the reference arm under torchrun (rank 0 alone
prints, the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = [3.0, 5.0][rank]
        m = bench.reduce_max(local_ms, world, "cpu")
        v = bench.weak_throughput(world, 131072 * 128, 20, m)
        out.put((rank, m, v, bench.rank_graph_seed(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_world2_max_over_ranks_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0), (r1, m1, v1, s1) = res
    assert m0 == m1 == 5.0                       # the slower rank sets the time
    assert v0 == v1 == pytest.approx(2 * 131072 * 128 * 20 / 5e-3)
    assert s0 != s1                              # every rank has its own graph


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5, 1, "cpu") == 2.5
    assert bench.weak_throughput(1, 10, 4, 2.0) == pytest.approx(20000.0)
    assert bench.rank_graph_seed(0) == 2


def test_reference_arm_under_torchrun_world2():
    port = free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--cpu-sample", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                       # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
