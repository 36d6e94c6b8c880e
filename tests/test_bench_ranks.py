"""The multi-rank bookkeeping of bench.py on CPU: two gloo ranks with different step
times report the slowest rank's time and the whole job's bytes over it, and a
reference-arm run on a non-zero rank does no work."""
from __future__ import annotations

import importlib.util
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        ms = [4.0, 7.5][rank]                       # rank 1 is the slow one
        slowest = b.max_over_ranks(ms, world, device="cpu")
        value = b.job_gbs(world, 10 ** 9, slowest)
        skipped = b.run_reference(None, None, 16, rank, world) if rank else None
        out.put((rank, slowest, value, skipped))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_bytes():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value, skipped in got:
        assert slowest == 7.5                       # max over ranks, on every rank
        assert abs(value - 2 * 1e9 / 7.5e-3 / 1e9) < 1e-9   # 2 ranks' bytes / slowest time
        if rank:
            assert skipped == 0                     # the reference arm runs on rank 0 only


def test_one_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(3.25, 1) == 3.25
    assert abs(b.job_gbs(1, 555188224, 0.0942) - 5893.7) < 0.1
