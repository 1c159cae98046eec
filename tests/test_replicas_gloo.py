"""Replica (data-parallel) timing logic of the decode benchmark, on 2 CPU ranks (gloo).

The decode step does not shard (each GPU decodes its own sequence); the only
cross-rank steps are the barriers around the timed region and the maximum of the
ranks' device times.  These run here as two gloo processes on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_scaffold_quantized_b200 import replicas as RP  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        RP.barrier(world)
        # rank r "measured" (10 + r) ms timed and (20 - r) ms end to end
        ms, ms_e2e = RP.max_over_ranks([10.0 + rank, 20.0 - rank], world)
        RP.barrier(world)
        out.put((rank, ms, ms_e2e, RP.job_tokens_per_s(64, 1, world, ms)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, ms_e2e, tok_s in results:
        assert ms == 11.0 and ms_e2e == 20.0          # elementwise max over the ranks
        assert tok_s == pytest.approx(2 * 64 / 0.011)  # all ranks' tokens over the slowest time


def test_single_rank_needs_no_process_group():
    assert RP.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
    RP.barrier(1)
    assert RP.job_tokens_per_s(512, 1, 1, 1000.0) == pytest.approx(512.0)
    with pytest.raises(ValueError):
        RP.job_tokens_per_s(1, 1, 1, 0.0)


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup, gpus, impl, no_cpu_baseline = 1, 3, 2, "reference", True

    assert bench.run_reference(Args, 1, 2) is None     # non-zero ranks exit without work
