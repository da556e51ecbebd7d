"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The decode path shards over (batch, KV head) with no exchange, so N GPUs run
N independent replicas; the only collectives are the timing barrier and the
max-over-ranks reduction of the elapsed time.  These tests run that plumbing
as two gloo ranks on the host.
"""
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
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    w, r, _ = bench.setup_dist(None)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    m = bench.max_over_ranks(1.5 + rank, w)
    from token_level_sparse_kv_b200.inputs import Workload

    class A:
        workload, batch, topk = "gqa_4k_b1", None, None

    wl = bench.workload_of(A)
    seeded = Workload(**{**wl.__dict__, "seed": wl.seed + 1000 * rank})
    q.put((rank, m, seeded.seed))
    dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [2.5, 2.5]  # every rank sees the max
    assert got[0][2] != got[1][2]  # replicas draw different data


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "gqa_4k_b1", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_bench_flushes_l2_only_for_steps_that_fit():
    """Steps whose bytes fit in the L2 are timed with a flush before each one
    (and config.l2 says so); the 1 GiB headline step streams past it."""
    sys.path.insert(0, ROOT)
    import bench
    from token_level_sparse_kv_b200.inputs import WORKLOADS

    l2 = 126 * 2**20
    assert bench.flushes_l2(WORKLOADS["gqa_4k_b1"], l2)
    assert bench.flushes_l2(WORKLOADS["gqa_32k_b4"], l2)
    assert not bench.flushes_l2(WORKLOADS["gqa_128k_b16"], l2)
    assert not bench.flushes_l2(WORKLOADS["hybrid_global_128k_b8"], l2)
    c = bench.config_of(WORKLOADS["gqa_4k_b1"], 1, flush=True)
    assert c["l2"].startswith("L2 flushed before every timed step")
    c = bench.config_of(WORKLOADS["gqa_128k_b16"], 1)
    assert c["l2"].startswith("inputs larger than L2")
