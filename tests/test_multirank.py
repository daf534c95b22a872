"""The N > 1 host path of bench.py on CPU: two gloo ranks.

bench.py under torchrun runs one independent replica of the step per rank
(the (sequence, head) units need no exchange), takes the slowest rank's
device time and reports the whole-job throughput.  These tests run that
aggregation with world_size 2 over gloo, and check that the reference arm
leaves every rank but 0 idle.
"""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 30.25][rank]  # the slower rank decides
        mx = bench.max_over_ranks(ms, dist, "cpu")
        e2e = bench.max_over_ranks([40.0, 35.0][rank], dist, "cpu")
        q.put((rank, mx, e2e, bench.job_value(world, 10, 4576, mx)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29000 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, e2e, value in out:
        assert mx == 30.25 and e2e == 40.0
        assert value == pytest.approx(2 * 10 * 4576 / 0.03025)


def test_job_value_single_rank_is_tokens_per_second():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0
    assert bench.job_value(1, 200, 4576, 100.0) == pytest.approx(200 * 4576 / 0.1)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_json_line():
    """Rank 0 of the reference arm prints one JSON line: the oracle timed on
    the host cores, with the keys of the bench contract (bounded samples, so
    this takes some 20 s)."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["unit"] == "tokens/s" and d["config"]["tokens_per_step"] == 4576
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert isinstance(cb["sample"], str) and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
