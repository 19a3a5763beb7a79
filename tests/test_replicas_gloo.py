"""Multi-process (world size 2, gloo on CPU) checks of the replica logic that
bench.py runs under torchrun: every rank sees the slowest rank's time, the
whole-job throughput counts the units of all ranks over that time, and the
reference arm runs on rank 0 only."""
import contextlib
import io
import json
import os
import socket
import sys
import multiprocessing as mp
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)


def _timing_worker(rank, world, port, q):
    _env(rank, world, port)
    import bench
    r, ws, dist = bench.dist_setup()
    local = [0.25, 0.75][r]           # rank 1 is the slow one
    slowest = bench.max_over_ranks(local, dist)
    bench.barrier(dist)
    q.put((r, ws, dist.get_backend(), slowest, bench.replica_value(ws, 16384, 10, slowest)))
    dist.destroy_process_group()


def _reference_worker(rank, world, port, q):
    _env(rank, world, port)
    import bench
    from learned_token_pruning_b200 import synth
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(types.SimpleNamespace(steps=1, warmup=0), synth.tiny_f32())
    q.put((rank, out.getvalue()))


def _run(worker, world=2, timeout=180):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=timeout) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(results)


def test_two_replicas_share_the_slowest_time():
    res = _run(_timing_worker)
    assert [r[0] for r in res] == [0, 1]
    for rank, ws, backend, slowest, value in res:
        assert ws == 2 and backend == "gloo"
        assert slowest == 0.75                       # max over ranks, seen by both
        assert value == pytest.approx(2 * 16384 * 10 / 0.75)


def test_replica_value_is_whole_job_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.replica_value(1, 100, 5, 2.0) == 250.0
    assert bench.replica_value(4, 100, 5, 2.0) == 1000.0   # weak scaling: four times the units, same time


def test_reference_arm_runs_on_rank_zero_only():
    res = _run(_reference_worker)
    (r0, out0), (r1, out1) = res
    assert out1 == ""                                  # rank 1 exits without work
    line = json.loads(out0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
