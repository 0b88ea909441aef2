"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks (no GPU).

The data path of the layer shards by token batch with no collective; the
benchmark's only cross-rank steps are the barrier and the max of the step
times, which these tests exercise."""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        mine = [10.0 + rank, 20.0 - rank, 1.0 * rank]          # per-rank times differ
        got = bench.reduce_max_over_ranks(dist, mine, torch.device("cpu"))
        dist.barrier()
        ref = bench.run_reference(type("A", (), {"oracle_tokens": 1, "warmup": 0, "steps": 1,
                                                 "workload": "tiny_f32", "tokens": 0, "experts": 0})(),
                                  rank, world) if rank != 0 else "skipped"
        out.put((rank, got, ref))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (g, ref)) for r, g, ref in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert res[r][0] == [11.0, 20.0, 1.0]        # every rank sees the max of each value
    assert res[1][1] is None                          # the reference arm runs on rank 0 only
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.job_value(2, 4096, 2.0) == pytest.approx(2 * 4096 / 2e-3)
    assert bench.job_value(1, 64, 0.5) == pytest.approx(64 / 5e-4)
