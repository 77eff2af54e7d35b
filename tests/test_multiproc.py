"""Multi-process paths of the benchmark on CPU (gloo, world size 2).

The layer itself is replicated, not sharded (one independent token stream
per GPU), so the only cross-rank steps are the barrier and the max-over-ranks
of the timings, and the reference arm's rank-0-only output.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        dist.barrier()
        q.put((rank, bench.max_over_ranks(1.5 + rank), bench.max_over_ranks(10.0 - rank)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2.5, 10.0), (1, 2.5, 10.0)]


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25


def test_replica_token_streams_differ():
    sys.path.insert(0, ROOT)
    import bench
    a = bench.make_inputs("reduced_e32_t1", 3, 1, "cpu", rank=0)
    b = bench.make_inputs("reduced_e32_t1", 3, 1, "cpu", rank=1)
    a2 = bench.make_inputs("reduced_e32_t1", 3, 1, "cpu", rank=0)
    assert all((x == y).all() for x, y in zip(a, a2))        # seeded: reproducible
    assert not any((x == y).all() for x, y in zip(a, b))     # rank 1 runs its own stream


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "reduced_e32_t1", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_bench_spawns_its_own_ranks_without_a_launcher():
    """`bench.py --gpus 2` started plainly (no WORLD_SIZE) runs two ranks
    itself under torch.distributed.run; rank 0 alone prints one line with
    n_gpus = 2 (the reference arm needs no GPU, so this runs on CPU)."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "reduced_e32_t1", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["metric"].startswith("reduced MoE-layer decode")


def test_every_workload_line_names_its_own_metric():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    names = [w for w in workloads.WORKLOADS]
    metrics = {bench.metric_for(w) for w in names}
    assert len(metrics) == len(names)  # no two workloads share a metric string
    assert bench.metric_for("decode_e512_t1") == bench.METRIC
    assert "T=2048" in bench.metric_for("prefill_e512_t2048_zipf")
    assert "T=4" in bench.metric_for("verify_e512_t4")
