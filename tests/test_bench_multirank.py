"""The multi-rank timing of bench.py on CPU: two gloo ranks (one process each)
report different times; every rank must see the slowest one, and the job's
throughput is the bytes of both ranks over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [12.5, 20.0][rank]
        ms_max = bench.max_over_ranks(ms, world, torch.device("cpu"))
        gbs = bench.aggregate_gbs(world, 1 << 30, 10, ms_max)
        q.put((rank, ms_max, gbs))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms_max, gbs in got:
        assert ms_max == 20.0
        assert gbs == pytest.approx(2 * (1 << 30) * 10 / 0.020 / 1e9)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.aggregate_gbs(1, 2e9, 4, 1000.0) == pytest.approx(8.0)
