"""The N > 1 host logic of bench.py on CPU: world_size-2 gloo ranks.

Every rank runs the same workload (independent problems, no data-path collective);
the only collective is the timing reduction: every rank gets the slowest rank's time,
and the whole-job rate counts every rank's work over that time.  The reference arm
runs on rank 0 only."""

import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import _multirank

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_take_the_slowest_time_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms = [3.0, 5.0]
    port = _free_port()
    procs = [ctx.Process(target=_multirank.rank_main, args=(r, 2, port, ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        rank, times, rate = q.get(timeout=120)
        got[rank] = (times, rate)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        times, rate = got[r][0], got[r][1]
        assert times == [5.0, 50.0]                 # element-wise max over the ranks
        assert abs(rate - 2.0 * 2.0e12 / 5e-3 / 1e12) < 1e-9


def test_one_rank_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], None) == [1.5, 2.5]
    assert bench.job_rate(1e12, 1, 1.0) == 1000.0


def _reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", str(world), "--steps", "1", "--warmup", "0", "--n", "256",
                           "--cpu-rows", "8"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference(0, 2)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
