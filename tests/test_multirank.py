"""The N > 1 path of bench.py on CPU: two gloo ranks, as torchrun would start
them.  Replicas only: no data-path collective exists, so what is shared across
ranks is the timing (the slowest rank's time) and the whole-job rate."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank: int, world: int, port: int, out):
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms = [1.5, 2.25][rank]                     # each rank's own device time
        slowest = bench.max_over_ranks(ms, world)
        rate = bench.job_rate(100, world, slowest)
        ref = bench.run_reference(type("A", (), dict(workload=bench.WORKLOAD, warmup=0,
                                                     steps=0))(), rank, world,
                                  None) if rank else None
        dist.barrier()
        out.put((rank, slowest, rate, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_the_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, rate, ref in res:
        assert slowest == 2.25                     # max over ranks, on every rank
        assert rate == pytest.approx(200 / 2.25e-3)   # 100 units per rank, 2 ranks
        if rank:
            assert ref is None                     # the reference arm runs on rank 0 only


def test_one_rank_is_unchanged():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.job_rate(64, 1, 2.0) == pytest.approx(32000.0)
