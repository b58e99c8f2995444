"""PeerAllreduce's host side on CPU with gloo, world sizes 2 to 4.

The library is replaced by a stand-in whose memory is POSIX shared memory (so
an address in one process maps another process's buffer after the handle
exchange, as CUDA IPC does) and whose "kernel" runs the peer protocol in
Python, each process its own rank, concurrently: phase A stores the oracle's
stage-1 tiles of every shard into the owner's mailbox slot and raises the
owner's flag; phase B waits for every rank's flag of its own shard, reduces
with the oracle and stores the result into every rank's gathered wire with a
flag; phase C waits for every shard's flag and decodes with the oracle.  This
checks the regions, the handle exchange, the pointer arrays, the epochs over
repeated calls and sizes, and the timeout report when a rank never runs.
Every rank's result must equal the oracle's all-reduce bit for bit."""
import os
import socket
import time
from multiprocessing import shared_memory

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as O


class ShmOps:
    """A stand-in for the library's peer calls over shared memory."""

    def __init__(self):
        self.blocks = {}
        self.next = 1 << 40

    def _add(self, shm):
        base = self.next
        self.next += 1 << 36
        self.blocks[base] = shm
        return base

    def view(self, addr):
        for base, shm in self.blocks.items():
            if base <= addr < base + shm.size:
                return np.ndarray((shm.size,), np.uint8, buffer=shm.buf)[addr - base:]
        raise KeyError(hex(addr))

    def alloc(self, nbytes):
        shm = shared_memory.SharedMemory(create=True, size=nbytes)
        np.ndarray((nbytes,), np.uint8, buffer=shm.buf)[:] = 0
        return self._add(shm)

    def export(self, addr):
        return self.blocks[addr].name.encode()

    def import_(self, handle):
        return self._add(shared_memory.SharedMemory(name=handle.decode()))

    def close(self, addr):
        self.blocks.pop(addr).close()

    def free(self, addr):
        shm = self.blocks.pop(addr)
        shm.close()
        shm.unlink()

    @staticmethod
    def mailbox_bytes(N, n, codec):
        T = n // 2048
        return N * -(-T // N) * O.tile_bytes(codec)

    @staticmethod
    def gather_bytes(n, codec):
        return n // 2048 * O.tile_bytes(codec)

    @staticmethod
    def flag_bytes(N, n):
        return 2 * N * 4                                   # one chunk per shard

    def _wait(self, addr, index, epoch, deadline, status, phase, rank):
        flags = self.view(addr)[:8 * 4 * 2].view(np.uint32)
        while int(flags[index]) < epoch:
            if time.monotonic() > deadline:
                status[:4] = torch.tensor([1, phase, rank, index], dtype=torch.int32)
                return False
            time.sleep(0.0005)
        return True

    def run(self, inputs, outputs, mailboxes, gathered, flags, n, codec, timeout_ns, status, rank0, ranks):
        assert ranks == 1 and inputs[rank0] is not None and all(x is None for i, x in enumerate(inputs) if i != rank0)
        epoch = int(status[4]) + 1
        if int(status[0]) == 0:
            self._run(inputs, outputs, mailboxes, gathered, flags, n, codec, timeout_ns, status, rank0, epoch)
        status[4] = epoch

    def _run(self, inputs, outputs, mailboxes, gathered, flags, n, codec, timeout_ns, status, rank0, epoch):
        N, r, T, tb = len(mailboxes), rank0, n // 2048, O.tile_bytes(codec)
        slot = -(-T // N)
        shard = [(j * T // N, (j + 1) * T // N) for j in range(N)]
        wire = O.quantize(inputs[r].view(torch.int16).numpy().view(np.uint16), codec)
        for j, (t0, t1) in enumerate(shard):                       # phase A
            self.view(mailboxes[j])[r * slot * tb:(r * slot + t1 - t0) * tb] = wire[t0 * tb:t1 * tb]
            self.view(flags[j])[:8 * N].view(np.uint32)[r] = epoch
        deadline = time.monotonic() + timeout_ns * 1e-9
        for s in range(N):                                         # phase B
            if not self._wait(flags[r], s, epoch, deadline, status, 1, r):
                return
        t0, t1 = shard[r]
        mine = self.view(mailboxes[r])
        red = O.reduce([mine[s * slot * tb:(s * slot + t1 - t0) * tb] for s in range(N)], 0, t1 - t0, codec)
        for q in range(N):
            self.view(gathered[q])[t0 * tb:t1 * tb] = red[:(t1 - t0) * tb]
            self.view(flags[q])[:8 * N].view(np.uint32)[N + r] = epoch
        for j in range(N):                                         # phase C
            if not self._wait(flags[r], N + j, epoch, deadline, status, 2, r):
                return
        dec = O.decode(self.view(gathered[r])[:T * tb].copy(), n, codec)
        outputs[r].copy_(torch.from_numpy(dec.view(np.int16).copy()).view(torch.bfloat16))


def inputs(N, n, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 2.0 ** r).to(torch.bfloat16) for r in range(N)]


def _worker(rank, world, port, codec, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_precision_all_b200.distributed import PeerAllreduce
        ops = ShmOps()
        ar = PeerAllreduce(ops=ops, timeout_ns=30_000_000_000, device=torch.device("cpu"))
        results = []
        for k, tiles in enumerate([5, 5, 12, 5]):                  # epochs 1, 2 on one region, then another size
            n = tiles * 2048
            x = inputs(world, n, 300 + k)[rank]
            out = ar.allreduce(x, codec)
            ar.check()
            results.append(out.view(torch.int16).numpy().copy())
        # below the threshold the message goes through the BF16 passthrough, in its own region
        n = 5 * 2048
        x = inputs(world, n, 400)[rank]
        out = ar.allreduce(x, codec, min_quant_bytes=2 * n + 2)
        ar.check()
        results.append(out.view(torch.int16).numpy().copy())
        epochs = ar.epochs()
        ar.release()
        assert not ops.blocks, "every mapping closed and the own regions freed"
        q.put((rank, results, epochs))
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        item = q.get(timeout=300)
        got[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world,codec", [(2, "int4"), (3, "int3"), (4, "fp8"), (2, "mxfp4"), (3, "bf16")])
def test_peer_allreduce_host_side(world, codec):
    got = spawn(_worker, world, codec)
    for k, tiles in enumerate([5, 5, 12, 5]):
        n = tiles * 2048
        ref, _ = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in inputs(world, n, 300 + k)],
                             codec)
        for r in range(world):
            assert np.array_equal(got[r][0][k].view(np.uint16), ref[0]), (codec, k, r)
    ref, used = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in inputs(world, 5 * 2048, 400)],
                            codec, 2 * 5 * 2048 + 2)
    assert used == "bf16"
    for r in range(world):
        assert np.array_equal(got[r][0][4].view(np.uint16), ref[0]), (codec, "threshold", r)
        want = {(5 * 2048, codec): 3, (12 * 2048, codec): 1}
        want[(5 * 2048, "bf16")] = want.get((5 * 2048, "bf16"), 0) + 1
        assert got[r][1] == want


def _absent_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_precision_all_b200 import lpar as L
        from quantized_precision_all_b200.distributed import PeerAllreduce
        ops = ShmOps()
        ar = PeerAllreduce(ops=ops, timeout_ns=300_000_000, device=torch.device("cpu"))
        n = 4 * 2048
        ar.region(n, "int4")                                       # both ranks map the regions
        err = None
        if rank == 0:                                              # rank 1 never makes the call
            ar.allreduce(inputs(world, n, 1)[0], "int4")
            try:
                ar.check()
            except L.PeerTimeout as e:
                err = str(e)
        status = ar.region(n, "int4").status.tolist()
        dist.barrier()
        ar.release()
        q.put((rank, err, status))
    finally:
        dist.destroy_process_group()


def test_peer_allreduce_reports_a_rank_that_never_runs():
    got = spawn(_absent_worker, 2)
    err, status = got[0]
    assert err is not None and "phase 1" in err, err
    assert status[:3] == [1, 1, 0] and status[3] == 1              # waiting for source 1's mailbox flag
    assert got[1][0] is None
