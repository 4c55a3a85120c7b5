"""Multi-process host logic of bench.py on the CPU (gloo, world size 2).

bench.py runs one independent replica of the workload per rank (no data-path
collective): only its barrier and the max-over-ranks reduction of the timed
region cross ranks, and only rank 0 prints the JSON line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    bench.barrier(w)
    got = bench.max_over_ranks(10.0 + r, w)
    q.put((r, w, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2, 11.0), (1, 2, 11.0)]


def test_reference_arm_two_ranks_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny", "--cpu-budget", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_head_shards_cover_the_problem():
    """--shard heads: each rank's workload holds heads/N heads, the line
    reports the problem's heads and strong scaling; a head count that does
    not split is refused."""
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    args = argparse.Namespace(workload="720p", heads=0, shard="heads")
    for world in (1, 2, 4, 8):
        w = bench.workload(args, world)
        assert w.heads * world == 40
        c = bench.config_of(w, world, shard="heads")
        assert c["heads"] == 40
        if world > 1:
            assert c["heads_per_gpu"] == 40 // world and "head-parallel" in c["parallelism"]
    assert bench.scaling_of(args) == "strong"
    assert bench.scaling_of(argparse.Namespace(shard="replicas")) == "weak"
    with pytest.raises(SystemExit):
        bench.workload(args, 3)
    # FLOPs: the shards' FLOPs add up to the problem's
    full = bench.workload(argparse.Namespace(workload="720p", heads=0, shard="replicas"), 4)
    assert 4 * bench.workload(args, 4).unmasked_flops() == full.unmasked_flops()


def test_reference_arm_head_shards_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny", "--cpu-budget", "1", "--shard", "heads"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["scaling"] == "strong" and lines[0]["config"]["heads"] == 2
    assert lines[0]["config"]["heads_per_gpu"] == 1

