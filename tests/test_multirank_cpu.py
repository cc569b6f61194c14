"""The N > 1 host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The delta path has no data exchange (every rank runs an independent replica
on its own batches), so the only cross-rank steps are the barrier around the
timed region and the max over ranks of the step time; the whole-job value is
every rank's tokens over the slowest rank's time.  The reference arm runs on
rank 0 alone and the other ranks leave without work."""

import contextlib
import io
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.sync_ranks(world)
        ms = bench.reduce_max(1.0 + rank, world)          # the slowest rank sets the step time
        value = bench.job_value(64, world, ms)
        bench.sync_ranks(world)
        out.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 2.0
        assert value == pytest.approx(64 * 2 / 2e-3)


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_value(512, 1, 2.0) == pytest.approx(512 / 2e-3)


def _reference_line(monkeypatch, rank, world):
    monkeypatch.setenv("RANK", str(rank))
    monkeypatch.setenv("WORLD_SIZE", str(world))
    monkeypatch.setenv("LOCAL_RANK", str(rank))
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--gpus", str(world), "--steps", "3",
                    "--warmup", "3"])
    return buf.getvalue().strip()


def test_reference_arm_rank0_prints_one_line_and_others_exit(monkeypatch):
    line = _reference_line(monkeypatch, 0, 2)
    d = json.loads(line)
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "tokens/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0
    assert _reference_line(monkeypatch, 1, 2) == ""
