"""The cross-GPU all-reduce on two or more GPUs, one process per GPU (skipped
when fewer than two GPUs are visible).

- PeerAllreduce (one peer-memory kernel per rank over CUDA IPC) and
  DistributedAllreduce (stage kernels with NCCL exchanges) must give every
  rank the oracle's all-reduce of all ranks' messages, bit for bit, over
  several calls and codecs.
- A rank that never makes its call (it leaves between steps, with nothing in
  flight): the other rank's waits give up after the timeout, `check()` raises
  PeerTimeout naming the phase that gave up first, and the process carries on.

Children run with NCCL's NVLink SHARP off (NCCL_NVLS_ENABLE=0) and a short
process-group timeout."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from oracle import oracle as O

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                                 reason="needs two or more GPUs")]


def inputs(N, n, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 2.0 ** r).to(torch.bfloat16) for r in range(N)]


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _init(rank, world, port, backend):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(rank)
    kw = {"device_id": torch.device("cuda", rank)} if backend == "nccl" else {}
    dist.init_process_group(backend, rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60), **kw)
    return dist


CASES = [(5, "int4"), (12, "int3"), (7, "fp8"), (9, "mxfp4"), (4, "bf16")]


def _worker(rank, world, port, kind, q):
    dist = _init(rank, world, port, "nccl" if kind == "nccl" else "gloo")
    try:
        from quantized_precision_all_b200.distributed import DistributedAllreduce, PeerAllreduce
        ar = PeerAllreduce() if kind == "peer" else DistributedAllreduce(chunks=2)
        got = []
        for k, (tiles, codec) in enumerate(CASES):
            x = inputs(world, tiles * 2048, 300 + k)[rank].cuda()
            y = ar.allreduce(x, codec)
            torch.cuda.synchronize()
            if kind == "peer":
                ar.check()
            got.append(_bits(y))
        dist.barrier()
        ar.release()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def _absent_worker(rank, world, port, q):
    dist = _init(rank, world, port, "gloo")
    try:
        from quantized_precision_all_b200 import lpar as L
        from quantized_precision_all_b200.distributed import PeerAllreduce
        ar = PeerAllreduce(timeout_ns=200_000_000)
        n = 6 * 2048
        ar.region(n, "int4")                                   # both ranks map the regions
        err = None
        if rank == 0:                                          # rank 1 leaves before the call
            ar.allreduce(inputs(world, n, 1)[0].cuda(), "int4")
            torch.cuda.synchronize()
            try:
                ar.check()
            except L.PeerTimeout as e:
                err = str(e)
        dist.barrier()
        ar.release()
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(target, world, *args):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, v = q.get(timeout=300)
        got[r] = v
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("kind", ["peer", "nccl"])
def test_cross_gpu_allreduce_matches_the_oracle(kind):
    world = min(torch.cuda.device_count(), 4)
    got = _spawn(_worker, world, kind)
    for k, (tiles, codec) in enumerate(CASES):
        xs = inputs(world, tiles * 2048, 300 + k)
        ref, _ = O.allreduce([_bits(x) for x in xs], codec)
        for r in range(world):
            assert np.array_equal(got[r][k], ref[0]), (kind, codec, r)


def test_peer_allreduce_reports_a_rank_that_never_calls():
    got = _spawn(_absent_worker, 2)
    assert got[0] is not None and ("phase 1" in got[0] or "phase 2" in got[0]), got
    assert got[1] is None
