"""PeerAllreduce's host side on CPU with gloo, world sizes 2 to 4.

The library's calls are replaced by a stand-in whose memory is POSIX shared
memory (so an address in one process maps another process's buffer after the
handle exchange, as CUDA IPC does) and whose "kernel" runs the peer protocol in
Python, with the library's buffer sizes and the kernel's chunk geometry and
flag indices, each process its own rank, concurrently: phase A stores the
oracle's stage-1 tiles of every chunk into the owner's mailbox slot and raises
the owner's flag for that chunk; phase B waits for every rank's flag of each
chunk of its own shard, reduces it with the oracle and stores the result into
every rank's gathered wire with a flag; phase C waits for every chunk's flag
and decodes with the oracle.  This
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
    """A stand-in for the library's peer calls over shared memory; `jitter`
    seeds random pauses between chunks (to vary the interleavings)."""

    def __init__(self, jitter=None):
        self.blocks = {}
        self.next = 1 << 40
        self.rng = np.random.default_rng(jitter) if jitter is not None else None

    def _pause(self):
        if self.rng is not None and self.rng.random() < 0.3:
            time.sleep(float(self.rng.random()) * 0.003)

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

    # the library's buffer sizes (host functions, no GPU needed): the stand-in lays its
    # buffers out as the kernel does
    @staticmethod
    def mailbox_bytes(N, n, codec):
        from quantized_precision_all_b200 import lpar as L
        return L.lpar_peer_mailbox_bytes(N, n, codec)

    @staticmethod
    def gather_bytes(n, codec):
        from quantized_precision_all_b200 import lpar as L
        return L.lpar_peer_gather_bytes(n, codec)

    @staticmethod
    def flag_bytes(N, n):
        from quantized_precision_all_b200 import lpar as L
        return L.lpar_peer_flag_bytes(N, n)

    def _flags(self, addr, words):
        return self.view(addr)[:4 * words].view(np.uint32)

    def _wait(self, flags, index, epoch, deadline, status, phase, rank):
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

    def _run(self, inputs, outputs, mailboxes, gathered, flags, n, codec, timeout_ns, status, me, epoch):
        """The kernel's protocol, chunk by chunk, with its geometry and flag indices:
        shard j = tiles [jT/N, (j+1)T/N), cut into P chunks [cS/P, (c+1)S/P); rank r's
        flags: s*P + c for source s's mailbox chunk c, N*P + j*P + c for owner j's
        gathered chunk c."""
        N, T, tb = len(mailboxes), n // 2048, O.tile_bytes(codec)
        P = self.flag_bytes(N, n) // (2 * N * 4)
        slot = -(-T // N)
        shard = [(j * T // N, (j + 1) * T // N) for j in range(N)]

        def chunk(j, c):
            b, e = shard[j]
            return b + c * (e - b) // P, b + (c + 1) * (e - b) // P

        wire = O.quantize(inputs[me].view(torch.int16).numpy().view(np.uint16), codec)
        for c in range(P):                                         # phase A, chunk-major
            for j in range(N):
                lo, hi = chunk(j, c)
                if lo == hi:
                    continue
                base = shard[j][0]
                self.view(mailboxes[j])[(me * slot + lo - base) * tb:(me * slot + hi - base) * tb] = \
                    wire[lo * tb:hi * tb]
                self._flags(flags[j], 2 * N * P)[me * P + c] = epoch
                self._pause()
        deadline = time.monotonic() + timeout_ns * 1e-9
        mine = self._flags(flags[me], 2 * N * P)
        base = shard[me][0]
        box = self.view(mailboxes[me])
        for c in range(P):                                         # phase B: my shard
            lo, hi = chunk(me, c)
            if lo == hi:
                continue
            for s in range(N):
                if not self._wait(mine, s * P + c, epoch, deadline, status, 1, me):
                    return
            wires = [box[(s * slot + lo - base) * tb:(s * slot + hi - base) * tb] for s in range(N)]
            red = O.reduce(wires, 0, hi - lo, codec)[:(hi - lo) * tb]
            for q in range(N):
                self.view(gathered[q])[lo * tb:hi * tb] = red
                self._flags(flags[q], 2 * N * P)[N * P + me * P + c] = epoch
            self._pause()
        for c in range(P):                                         # phase C: every shard
            for j in range(N):
                lo, hi = chunk(j, c)
                if lo < hi and not self._wait(mine, N * P + j * P + c, epoch, deadline, status, 2, me):
                    return
        dec = O.decode(self.view(gathered[me])[:T * tb].copy(), n, codec)
        outputs[me].copy_(torch.from_numpy(dec.view(np.int16).copy()).view(torch.bfloat16))


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
    from quantized_precision_all_b200 import lpar as L
    P = L.lpar_peer_flag_bytes(2, 4 * 2048) // (2 * 2 * 4)
    assert status[:3] == [1, 1, 0] and status[3] == P              # source 1's mailbox flag of chunk 0
    assert got[1][0] is None


def _stress_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_precision_all_b200.distributed import PeerAllreduce
        ar = PeerAllreduce(ops=ShmOps(jitter=1000 + rank), timeout_ns=60_000_000_000, device=torch.device("cpu"))
        results = []
        for k in range(8):                                     # epochs 1..4 on each of two regions
            codec = ("int4", "fp8")[k % 2]
            x = inputs(world, 40 * 2048, 700 + k)[rank]
            results.append(ar.allreduce(x, codec).view(torch.int16).numpy().copy())
            ar.check()
        epochs = ar.epochs()
        ar.release()
        q.put((rank, results, epochs))
    finally:
        dist.destroy_process_group()


def test_peer_protocol_under_random_interleavings():
    """Three ranks pausing at random between chunks (each its own seed), eight calls
    over two regions: every result equals the oracle's, the epochs count the calls."""
    world = 3
    got = spawn(_stress_worker, world)
    for k in range(8):
        codec = ("int4", "fp8")[k % 2]
        ref, _ = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in inputs(world, 40 * 2048, 700 + k)],
                             codec)
        for r in range(world):
            assert np.array_equal(got[r][0][k].view(np.uint16), ref[0]), (k, r)
    for r in range(world):
        assert got[r][1] == {(40 * 2048, "int4"): 4, (40 * 2048, "fp8"): 4}
