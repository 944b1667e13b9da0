"""Host-side logic of bench.py, on CPU: the replica aggregation over two gloo ranks and the
reference arm (the CPU oracle) printing its JSON line on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _ranks_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        secs, nbytes = bench.aggregate(1.0 + rank, 10.0 * (rank + 1), torch.device("cpu"))
        m = bench.dist_max(3.0 - rank, torch.device("cpu"))
        bench.barrier()
        out.put((rank, secs, nbytes, m))
    finally:
        dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    """A replica job's time is the slowest rank's and its work the sum over ranks."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_ranks_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, secs, nbytes, m in got:
        assert secs == 2.0 and nbytes == 30.0 and m == 3.0


def test_aggregate_single_process_is_identity():
    assert bench.aggregate(1.5, 7.0, torch.device("cpu")) == (1.5, 7.0)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args,
                          capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)


def test_reference_arm_line():
    """--impl reference times the oracle and prints one JSON line on the qg arm's metric, unit,
    direction and config."""
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-seconds", "2"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["config"] == bench.bench_config(1)
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] == 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_gpus_flag_launches_replica_ranks():
    """--gpus 2 without a launcher starts two ranks under torch.distributed.run (rendezvous on
    127.0.0.1; the reference arm joins a gloo group on every rank), and rank 0 alone prints."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--steps", "1", "--warmup", "3", "--ref-seconds", "1"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["config"] == bench.bench_config(2)


def test_gpus_flag_must_match_the_launcher():
    """Under a launcher, --gpus must equal WORLD_SIZE (no silent single-rank run)."""
    r = _run_bench(["--gpus", "4", "--impl", "reference", "--steps", "1"],
                   {"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode == 2 and "WORLD_SIZE" in r.stderr
