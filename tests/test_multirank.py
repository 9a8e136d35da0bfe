"""The multi-GPU path of bench.py on CPU: two gloo ranks in separate
processes.  The path shards by replica (each rank its own batch) with no
data-path collective; what crosses ranks is the barrier and the
max-over-ranks timing, checked here, plus the rule that only rank 0 runs and
prints the reference arm."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow replica
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        torch.distributed.barrier()
        out.put((rank, ms, bench.job_value(ms, 3, world), bench.replica_seeds(rank)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_replica():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, s0), (r1, ms1, v1, s1) = res
    assert ms0 == ms1 == 15.0                        # max over ranks
    assert v0 == v1 == pytest.approx(3 * 64 * 2 / 0.015)   # all ranks' steps / slowest time
    assert len(set(s0) | set(s1)) == 6               # independent replica streams


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_value(1000.0, 2, 1) == pytest.approx(128.0)


def _run_bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    p = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"},
                   "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3")
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_line():
    p = _run_bench({"RANK": "0", "WORLD_SIZE": "1", "LOCAL_RANK": "0"},
                   "--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-budget", "4")
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_clock_samples_parse_reasons_and_median():
    import bench
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1950, 1965, 980.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1965, 1965, 990.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    got = bench.parse_clock_samples(lines)
    assert got == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                   "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 3}
    assert bench.parse_clock_samples([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                                             "samples": 0}
