"""N>1 host logic of bench.py on CPU: world_size-2 gloo ranks.

Each rank runs an independent replica (no collective on the data path); the
only collectives are the timing reduction (max over ranks) and barriers. The
reference arm runs on rank 0 only; other ranks exit without work.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms)
        dist.barrier()
        v = bench.weak_scaling_gbs(world, 1_000_000, 10, ms)
        q.put((rank, ms, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, v in out:
        assert ms == 5.0  # every rank sees the slowest rank's time
        # 2 ranks x 1 MB x 10 steps in 5 ms = 4 GB/s whole-job
        assert abs(v - 4.0) < 1e-9


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.5) == 2.5
    assert abs(bench.weak_scaling_gbs(1, 2_000_000, 4, 8.0) - 1.0) < 1e-12


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
