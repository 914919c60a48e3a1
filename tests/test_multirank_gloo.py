"""The benchmark's multi-rank plumbing, run as two gloo ranks on CPU (the
same code path torchrun drives with NCCL on GPUs): every rank reports its
own time, the job takes the slowest rank's time, the whole-job value counts
the units of all ranks, and the reference arm runs on rank 0 alone."""
from __future__ import annotations

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))


def _plumbing(rank, world, port, q):
    _env(rank, world, port)
    import torch.distributed as dist

    import bench
    r, w, _ = bench.dist_init("gloo")
    ms = 10.0 + 5.0 * r                   # rank 1 is the slow one
    m = bench.max_over_ranks(ms, w)
    bench.barrier(w)
    q.put((r, w, m, bench.job_value(64 * 100, m, w)))
    dist.destroy_process_group()


def _reference_arm(rank, world, port, q):
    _env(rank, world, port)
    import bench
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "2",
                "--warmup", "1"]
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    q.put((rank, buf.getvalue()))


def _run(target, world=2):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_two_ranks_take_the_slowest_time():
    out = _run(_plumbing)
    assert [o[0] for o in out] == [0, 1]
    for r, w, m, v in out:
        assert w == 2
        assert m == pytest.approx(15.0)                     # both ranks agree on the max
        assert v == pytest.approx(2 * 6400 / 0.015)         # units of both ranks / slowest time


def test_reference_arm_prints_on_rank_zero_only():
    out = _run(_reference_arm)
    lines0 = [l for l in out[0][1].splitlines() if l.startswith("{")]
    assert len(lines0) == 1 and out[1][1].strip() == ""
    d = json.loads(lines0[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
