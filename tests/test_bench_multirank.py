"""Host-side multi-rank logic of bench.py, run as world-size-2 gloo process groups on the
CPU: every rank gets the same workload shape on its own data (weak scaling), and the
step time reported is the max over ranks. Also checks the reference arm's rank rules."""

import json
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
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload("wan13b", rank, world)
        local_ms = 1.0 + rank * 0.25
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        seeds = [None] * world
        dist.all_gather_object(seeds, w.data_seed)
        out_q.put((rank, w.H, w.N, m, seeds))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_shards_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, H, N, m, seeds in results:
        assert (H, N) == (12, 32760)          # same workload shape on every rank
        assert m == 1.25                      # max over ranks, identical everywhere
        assert len(set(seeds)) == world       # each rank draws its own data


def test_single_rank_defaults():
    sys.path.insert(0, ROOT)
    import bench
    w = bench.rank_workload("wan13b", 0, 1)
    assert w.data_seed == 1 and w.H == 12
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
