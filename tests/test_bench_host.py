"""Host-side logic of bench.py's multi-process path, on CPU.

The path does not shard (one weight matrix per call), so bench.py --gpus N
runs N independent replicas: the ranks meet only for barriers and the
max-over-ranks reduction of the device time.  That reduction is checked here
with two gloo ranks; the reference arm (the CPU oracle) must run on rank 0
only and leave the other ranks without work.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist, r, w, local = bench._dist("gloo")
    try:
        assert (r, w, local) == (rank, world, rank)
        got = bench.max_over_ranks(values[rank], dist, "cpu")
        dist.barrier()
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    values = [1.25, 7.5]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, values, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(out.get(timeout=10) for _ in range(world))
    assert got == {0: max(values), 1: max(values)}


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


def _reference(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                           "--steps", "2", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _reference(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference(0)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
