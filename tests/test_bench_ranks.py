"""bench.py's multi-rank host logic on the CPU, world size 2 over gloo
(127.0.0.1): each rank reads its RANK / WORLD_SIZE / LOCAL_RANK, the job time
is the slowest rank's and the job's work the sum of every rank's (weak
scaling, no data-path collective), each rank seeds its own batch element, and
the reference arm leaves every rank but 0 silent."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

import bench
from _ranks import reduction_rank

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_take_max_time_and_summed_work():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=reduction_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    seen = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, env, ms, work, _ in seen:
        assert env == (rank, 2, rank)
        assert ms == 15.0         # the slower rank's time
        assert work == 300.0      # 100 + 200
    assert seen[0][4] != seen[1][4]   # distinct batch elements


def test_single_process_reduction_is_identity():
    assert bench._reduce_max_sum(12.5, 7.0, "cpu") == (12.5, 7.0)


def test_reference_arm_is_silent_off_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("mask", ["cluster", "psa"])
def test_reference_line_shape(mask):
    """Rank 0 of the reference arm prints one JSON line with the contract's keys
    (one bounded oracle sample, a few seconds of CPU), for either plan source."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--mask", mask, "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert ("PSA" in line["metric"]) == (mask == "psa")
