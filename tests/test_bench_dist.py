"""The bench's multi-process path on the CPU (gloo, world size 2): per-rank timings reduce to
the max, throughput aggregates over ranks (weak scaling), and only rank 0 prints.  The reference
arm exits quietly on ranks other than 0."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_distributed("gloo", timeout_s=60)
    try:
        mine = [10.0 + rank, 3.0 - rank, 7.5 if rank == 1 else 1.0]
        got = bench.max_over_ranks(mine, dist, "cpu")
        value = bench.aggregate_tflops(2.0e12, world, got[0])
        dist.barrier()
        out.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [11.0, 3.0, 7.5]          # max over ranks, element-wise
        assert abs(value - 2 * 2.0e12 / 11.0e-3 / 1e12) < 1e-9


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_distributed("gloo") is None or int(os.environ.get("WORLD_SIZE", "1")) > 1
    assert bench.max_over_ranks([1.5, 2.5], None, "cpu") == [1.5, 2.5]


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
