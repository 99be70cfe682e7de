"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduction, the per-rank batch, and the reference arm
launched the way the driver launches N > 1 (torch.distributed.run), where only
rank 0 works and prints."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.reduce_max(float(rank + 1) * 1.5, world)
        bench.barrier(world)
        order = bench.rank_token_order(64, rank)
        q.put((rank, m, order.tolist(), bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_rank_batches_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(2):
        r, m, order, env = q.get(timeout=120)
        res[r] = (m, order, env)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 3.0                     # max over ranks
    assert res[0][1] == list(range(64))                      # rank 0 keeps the batch
    assert sorted(res[1][1]) == list(range(64)) and res[1][1] != list(range(64))
    assert res[1][2] == (1, 2, 1)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "fixture",
           "--steps", "3", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                                   # only rank 0 prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_rejects_multi_gpu_without_launcher():
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--impl", "reference",
                          "--workload", "fixture"], cwd=ROOT, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode != 0
    assert "torch.distributed.run" in out.stderr


def test_traffic_hash_ignores_comments_only():
    """A recorded ncu traffic figure stays valid across comment edits of the
    kernel sources and is dropped by any code edit."""
    sys.path.insert(0, ROOT)
    import bench
    src = 'int a = 1; // one\n/* block\n comment */ const char* s = "x//y /*z*/";\n\nint b;\n'
    assert bench.strip_c_comments(src) == 'int a = 1;\n const char* s = "x//y /*z*/";\nint b;'
    assert bench.strip_c_comments(src.replace("// one", "// two")) == bench.strip_c_comments(src)
    assert bench.strip_c_comments(src.replace("b;", "c;")) != bench.strip_c_comments(src)
    assert bench.strip_c_comments("char q = '\"'; // x") == "char q = '\"';"


def test_cpulist_parsing_and_affinity_restore():
    """sysfs cpulists ("0-3,8,10-11"); the near-GPU allocation scope restores the
    process's CPU affinity, and does nothing when the GPU's node is unknown."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}
    before = os.sched_getaffinity(0)
    near = bench.NearGpuHostMemory.__new__(bench.NearGpuHostMemory)
    near.cpus, near.saved = {min(before)}, None
    with near:
        assert os.sched_getaffinity(0) == {min(before)}
    assert os.sched_getaffinity(0) == before
    near.cpus, near.saved = None, None
    with near:
        assert os.sched_getaffinity(0) == before
    assert "unknown" in near.describe()
