"""The cross-process all-reduce (quantized_precision_all_b200.distributed) on CPU
with gloo, world sizes 2 to 4: the host orchestration (shard partition, the
all-to-all split sizes, rank order of the received wires, the padded
all-gather into one buffer and the per-shard decode) runs with the oracle's
stage functions, with the message in one chunk or several (the chunks' exchanges
issued asynchronously), and every rank's result must equal the oracle's
all-reduce of all ranks' messages bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as O


def oracle_stages():
    from quantized_precision_all_b200.distributed import Stages

    def bits(t):
        return t.view(torch.int16).numpy().view(np.uint16)

    def quantize(x, codec, wire):
        wire.copy_(torch.from_numpy(O.quantize(bits(x), codec).copy()))

    def reduce(wires, tiles, codec, out):
        if tiles:
            red = O.reduce([w.numpy() for w in wires], 0, tiles, codec)[:tiles * O.tile_bytes(codec)]
            out.copy_(torch.from_numpy(red.copy()))

    def decode(wire, n, codec, out):
        out.copy_(torch.from_numpy(O.decode(wire.numpy(), n, codec).view(np.int16).copy()).view(torch.bfloat16))

    return Stages(quantize, reduce, decode, O.tile_bytes)


def inputs(N, n, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 3.0 ** r).to(torch.bfloat16) for r in range(N)]


def _worker(rank, world, port, n, codec, thr, chunks, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_precision_all_b200.distributed import DistributedAllreduce
        xs = inputs(world, n, 77)
        ar = DistributedAllreduce(stages=oracle_stages(), chunks=chunks)
        out = ar.allreduce(xs[rank], codec, thr)
        # a second call reuses the cached exchange buffers
        again = ar.allreduce(xs[rank], codec, thr, out=torch.empty_like(out))
        assert torch.equal(out.view(torch.int16), again.view(torch.int16))
        q.put((rank, out.view(torch.int16).numpy().copy()))
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,tiles,codec,thr,chunks", [(2, 5, "int3", 0, 1), (3, 4, "int4", 0, 1),
                                                          (4, 3, "fp8", 0, 1), (3, 2, "mxfp4", 0, 1),
                                                          (4, 7, "bf16", 0, 1), (2, 3, "int3", 1 << 20, 1),
                                                          (3, 11, "int3", 0, 3), (4, 9, "int4", 0, 4),
                                                          (2, 3, "mxfp4", 0, 5)])
def test_cross_process_allreduce_equals_the_emulation(world, tiles, codec, thr, chunks):
    n = tiles * 2048
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, codec, thr, chunks, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    xs = inputs(world, n, 77)
    ref, _ = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in xs], codec, thr)
    for r in range(world):
        assert np.array_equal(got[r].view(np.uint16), ref[0]), (r, codec)
