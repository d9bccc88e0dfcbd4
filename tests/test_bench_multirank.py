"""bench.py's multi-rank host logic on CPU: two gloo ranks (no GPU).

Under torchrun every rank times the same workload on its own GPU. The job's
time is the slowest rank's, and the whole-job value adds the ranks' units. The
reference arm prints from rank 0 only.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank: int, world: int, port: int, local_ms: list, q) -> None:
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(local_ms[rank], world, "cpu")
        e = bench.max_over_ranks(local_ms[rank] * 2.0, world, "cpu")  # a second collective, same order
        q.put((rank, t, e, bench.whole_job_mvox(world, 10, 10, 209715, t)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_takes_the_slowest_rank_with_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    local = [3.0, 7.5]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, local, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in results) == [0, 1]
    for _, t, e, v in results:
        assert t == 7.5 and e == 15.0
        assert v == pytest.approx(2 * 10 * 10 * 209715 / 7.5e-3 / 1e6)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.25, 1, "cpu") == 4.25
    assert bench.whole_job_mvox(1, 2, 10, 1000, 20.0) == pytest.approx(1.0)


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line():
    """Single-rank reference arm: the oracle timed on host cores, one JSON line."""
    import json

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
