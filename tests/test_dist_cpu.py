"""The N>1 path of bench.py on CPU: two gloo ranks, barrier, max over ranks and
the whole-job throughput (each rank runs its own batch; no data-path
collective)."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.reduce_max(local_ms, world)
        agg = bench.aggregate(tokens_per_rank=64, steps=4, ms_max=ms, world=world)
        out.put((rank, ms, agg["value"], agg["ms_per_step"]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_is_max_and_value_is_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, ms_step in res:
        assert ms == 15.0  # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 64 * 4 / 0.015)  # all ranks' tokens over that time
        assert ms_step == pytest.approx(15.0 / 4)
