"""The benchmark's multi-rank host logic on CPU with two gloo ranks: the
max-over-ranks reduction of the step time, the weak-scaling aggregate, and
the reference arm running on rank 0 only."""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_us = [12.5, 17.0][rank]
        m = bench.max_over_ranks(step_us, "cpu")
        agg = bench.aggregate(m, world, 1_048_576)
        dist.barrier()
        q.put((rank, m, agg))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_aggregate():
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
    for rank, m, agg in res:
        assert m == 17.0
        assert agg["value"] == 17.0
        assert agg["keys_scored_per_s"] == pytest.approx(2 * 1_048_576 / 17e-6)


def test_reference_arm_is_silent_off_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), dict(workload="tiny_4k", steps=2, warmup=1))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""


def test_reference_arm_line_on_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = type("A", (), dict(workload="tiny_4k", steps=3, warmup=1))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    line = json.loads(buf.getvalue())
    assert line["impl"] == "reference" and line["unit"] == "µs/step"
    assert line["higher_is_better"] is False and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
