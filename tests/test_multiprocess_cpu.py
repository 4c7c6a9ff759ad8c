"""The multi-rank host logic of the benchmark on CPU: two gloo ranks, one process each.

The decode path shards by independent (batch, kv head) groups (weak scaling, no data exchange),
so the only collective is the timing reduction: every rank takes the job's time as the maximum
over ranks, and the job's throughput counts the tokens of all ranks over that time.
"""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        dist.barrier()
        total, e2e = bench.job_timing(10.0 + 5.0 * rank, 30.0 - 4.0 * rank, world,
                                      torch.device("cpu"))
        out.put((rank, total, e2e, bench.job_throughput(8, world, 100, total)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_sum_the_tokens():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:  # a rank that fails ends at once; a stuck one is ended by the 60 s timeout
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
            p.join()
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in procs)
    assert [r[0] for r in res] == [0, 1]
    for _, total, e2e, tput in res:
        assert total == 15.0 and e2e == 30.0          # max over ranks, every rank agrees
        assert tput == pytest.approx(8 * 2 * 100 / 0.015)


def test_single_rank_is_its_own_time():
    import torch
    import bench
    assert bench.job_timing(3.0, 4.0, 1, torch.device("cpu")) == (3.0, 4.0)
    assert bench.job_throughput(8, 1, 10, 2.0) == pytest.approx(8 * 10 / 0.002)


def _rank_dies_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    dist.barrier()
    if rank == 1:
        os._exit(3)  # leaves between steps, with no collective in flight
    try:
        bench.job_timing(1.0, 2.0, world, torch.device("cpu"))
        out.put((rank, "no error"))
    except Exception as e:  # the survivor learns of it from its next collective
        out.put((rank, type(e).__name__))


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
            p.join()
    assert procs[1].exitcode == 3
    rank, what = out.get(timeout=10)
    assert rank == 0 and what != "no error"
