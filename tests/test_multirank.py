"""bench.py's multi-rank logic on CPU: gloo ranks take the max over ranks and
count every rank's tokens; the reference arm runs on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks_and_job_throughput_gloo(world, monkeypatch):
    import torch.multiprocessing as mp
    monkeypatch.setenv("PYTHONPATH", os.pathsep.join([ROOT, TESTS, os.environ.get("PYTHONPATH", "")]))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    import multirank_worker
    procs = [ctx.Process(target=multirank_worker.run, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max([12.0, 15.5, 9.25, 14.0][:world])
    for rank, ms, value in results:
        assert ms == slowest
        assert value == pytest.approx(world * 64 * 10 / (slowest / 1e3))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.job_throughput(1, 64, 100, 500.0) == pytest.approx(12800.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
    assert buf.getvalue() == ""


def test_reference_arm_line_on_cpu(monkeypatch):
    """The oracle arm on a bounded sample of the small workload (CPU only)."""
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                           "--warmup", "3", "--cpu-sample", "8"]) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
