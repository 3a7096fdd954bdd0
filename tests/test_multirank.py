"""The benchmark's multi-rank logic on CPU: world_size-2 `gloo` ranks.

The path shards by (batch, head) with no data exchange, so the only
collectives are the timing reductions: every reported time is the max over
ranks, and the whole-job rate counts every rank's units against that time.
The reference arm runs on rank 0 alone; the other ranks exit without work.
"""
import os
import socket
import sys
import types

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, dist, "cpu")
        rate = bench.whole_job_rate(1000, world, 4, total)
        # the reference arm: rank 0 alone runs it; the others return 0 at once
        args = types.SimpleNamespace(workload="tiny", steps=1, warmup=0, gpus=world)
        ref_rc = bench.run_reference(args, rank, world) if rank != 0 else 0
        dist.barrier()
        out.put((rank, total, rate, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_every_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, rate, ref_rc in got:
        assert total == 15.0                     # max over ranks, seen by every rank
        assert rate == pytest.approx(1000 * 2 * 4 / 15e-3)
        assert ref_rc == 0
    assert [g[0] for g in got] == [0, 1]


def test_single_process_reductions_are_the_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_rate(10, 1, 2, 4.0) == pytest.approx(10 * 2 / 4e-3)
