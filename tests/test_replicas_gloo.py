"""Multi-process replica bookkeeping of bench.py on CPU: two `gloo` ranks (no GPU).

bench.py runs one decode replica per GPU with no collective on the data path; the ranks meet
only to take the slowest rank's time, and the job's throughput counts every rank's audio.
"""
from __future__ import annotations

import datetime
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 100.0 + 7.0 * r                      # each replica's own timed total
        mx = bench.max_over_ranks(ms, w, torch.device("cpu"))
        out[r] = (w, local, mx, bench.job_throughput(w, 4, 20.0, mx))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (w, local, mx, value) in res.items():
        assert (w, local) == (2, r)
        assert mx == 107.0                         # the max over ranks, on every rank
        assert value == pytest.approx(2 * 4 * 20.0 / 0.107)


def test_single_process_needs_no_collective(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    assert bench.job_throughput(1, 10, 20.0, 12.5) == pytest.approx(10 * 20.0 / 0.0125)
