"""Host logic of bench.py that needs no GPU.  Multi-GPU is replicas only
(the path has no exchange step, so N GPUs run N independent replicas): gloo
ranks on the CPU check the max-over-ranks timing and the whole-job rate, and
the reference arm's other ranks exit without work.  The reference arm's JSON
line is checked on a tiny layer."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        q.put((rank, bench.max_over_ranks(times[rank], world, "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_gives_every_rank_the_slowest_time(world):
    times = [12.5, 40.25, 7.0][:world]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {r: max(times) for r in range(world)}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def test_whole_job_rate_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    # 8200 tokens a step on each of 4 replicas, 10 steps in 20 ms (the slowest rank)
    assert bench.whole_job_rate(8200, 4, 10, 20.0) == pytest.approx(8200 * 4 * 10 / 0.020)
    assert bench.whole_job_rate(8200, 1, 10, 20.0) * 4 == pytest.approx(bench.whole_job_rate(8200, 4, 10, 20.0))


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """The reference arm (the float64 oracle on host cores) prints one JSON
    line with the contract's keys; a tiny layer keeps it quick here."""
    import json
    import types
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "WORKLOAD", dict(bench.WORKLOAD, S=64, hidden=128, n_heads=4, n_kv_heads=2,
                                                 head_dim=32, cap=80))
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.run_reference(types.SimpleNamespace(steps=2, warmup=3, gpus=1))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.WORKLOAD["name"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
