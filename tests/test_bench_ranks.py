"""The benchmark's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

bench.py runs one replica of the workload per rank (independent sequences,
no data-path collective). What the ranks share is host logic: the job's
time is the slowest rank's (one all-reduce of a scalar), the value counts
the units of all ranks, and only rank 0 prints the JSON line; with the
reference arm, ranks other than 0 exit without work. These tests run that
logic in two spawned processes over gloo, with no GPU.
"""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo")
    ms = bench.max_over_ranks(1.5 + r, w, device="cpu")   # rank r took 1.5 + r ms
    bench.barrier(w, sync_cuda=False)
    value = bench.job_value(w, 32768, ms)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.rank0_print(r, {"value": value, "ms_per_step": ms, "n_gpus": w})
    out.put((r, w, ms, value, buf.getvalue()))
    dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time_and_rank0_prints():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, w, ms, value, printed = out.get(timeout=120)
        results[r] = (w, ms, value, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        w, ms, value, _ = results[r]
        assert w == world
        assert ms == pytest.approx(2.5)                      # the slower rank's time
        assert value == pytest.approx(world * 32768 / 2.5e-3)  # units of all ranks
    line = json.loads(results[0][3])
    assert line["n_gpus"] == world and line["ms_per_step"] == pytest.approx(2.5)
    assert results[1][3] == ""                               # only rank 0 prints


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_value(1, 1000, 2.0) == pytest.approx(5e5)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, ref_budget = 5, 3, 8.0

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.bench_reference(Args()) is None
    assert buf.getvalue() == ""
