"""Multi-process (world size 2, gloo on CPU) checks of the bench's N-GPU
logic: each rank owns an independent batch (its own seed; no data-path
collective), the job time is the max over ranks, and the whole-job rate
counts every rank's sequences."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as tdist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings (ms): rank 1 is the slow one on the first value
        mine = [10.0 + 5.0 * rank, 3.0 - rank]
        got = bench.max_over_ranks(mine)
        out[rank] = (got, bench.rank_seed(0x5EED0001, rank),
                     bench.weak_scaling_rate(world, 4, 20, got[0]))
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_two_ranks_max_time_and_weak_scaling():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got0, seed0, rate0 = out[0]
    got1, seed1, rate1 = out[1]
    assert got0 == got1 == [15.0, 3.0]              # max over ranks, identical on every rank
    assert seed0 != seed1                            # independent batches
    assert rate0 == rate1 == pytest.approx(2 * 4 * 20 / 0.015)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.weak_scaling_rate(1, 4, 10, 1000.0) == 40.0
