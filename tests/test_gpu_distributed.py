"""The cross-process all-reduce with the library's CUDA stage kernels (needs a
B200): 2 to 4 processes share the one GPU, each runs lpar_quantize,
lpar_reduce and lpar_decode on its own device buffers, and the exchanges run
over gloo on host copies of the wire buffers.  No kernel of one process waits
for another process: every exchange happens on the host between launches.
Every rank's result must equal the oracle's all-reduce of all ranks' messages
bit for bit, on a first call and on a second call that reuses the cached
exchange buffers."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as O

pytestmark = pytest.mark.gpu


def inputs(N, n, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 3.0 ** r).to(torch.bfloat16) for r in range(N)]


def _worker(rank, world, port, n, codec, thr, chunks, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_precision_all_b200.distributed import DistributedAllreduce
        xs = inputs(world, n, 91)
        x = xs[rank].cuda()
        ar = DistributedAllreduce(chunks=chunks)
        assert ar._host(x.device)                       # gloo: the wire bytes travel through host copies
        out = ar.allreduce(x, codec, thr)
        again = ar.allreduce(x, codec, thr, out=torch.empty_like(out))
        torch.cuda.synchronize()
        q.put((rank, out.view(torch.int16).cpu().numpy().copy(), again.view(torch.int16).cpu().numpy().copy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,tiles,codec,thr,chunks", [(2, 9, "int3", 0, 1), (3, 10, "int4", 0, 3),
                                                          (4, 13, "fp8", 0, 2), (2, 7, "mxfp4", 0, 4),
                                                          (3, 5, "bf16", 0, 1), (2, 6, "int3", 1 << 20, 2)])
def test_cross_process_cuda_stages(world, tiles, codec, thr, chunks):
    n = tiles * 2048
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, codec, thr, chunks, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, a, b = q.get(timeout=300)
        got[r] = (a, b)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    xs = inputs(world, n, 91)
    ref, _ = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in xs], codec, thr)
    for r in range(world):
        assert np.array_equal(got[r][0].view(np.uint16), ref[0]), (r, codec)
        assert np.array_equal(got[r][1].view(np.uint16), ref[0]), (r, codec, "second call")
