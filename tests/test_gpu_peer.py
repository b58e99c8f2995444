"""The peer-memory all-reduce kernel (lpar_allreduce_peer) against the CPU
oracle, bit for bit (needs a B200).

All N ranks run in one launch on the one GPU, so every wait is on flags that
the same launch raises.  Besides the outputs, the exchange buffers are checked
against the oracle: rank j's mailbox slot s holds shard j of rank s's stage-1
wire, and every rank's gathered wire holds the requantised wire of the whole
message.  Every buffer the kernel writes has guard bands.  The failure path is
tested with a rank whose buffers are mapped host memory and which never runs:
its flags are never raised, the waits give up after the timeout and report it
in the status words, and the context stays usable.  The CUDA IPC calls are
tested across processes that share the GPU: each process exports its buffers,
one process maps them all and runs the launch, the others only read their
results afterwards (no kernel waits for another process)."""
import os
import socket
import time

import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as O
from tests.test_gpu_parity import Guarded, adversarial_bf16, host_u16, random_bf16, to_device

pytestmark = pytest.mark.gpu

CODECS = ("int4", "int3", "fp8", "mxfp4", "bf16")
TIMEOUT_NS = 2_000_000_000


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


class Bufs:
    """Guarded mailboxes, gathered wires and flags of N ranks, and the status."""

    def __init__(self, L, N, n, codec):
        self.N, self.n, self.codec = N, n, codec
        self.mbox = [Guarded(L.lpar_peer_mailbox_bytes(N, n, codec), fill=0) for _ in range(N)]
        self.gath = [Guarded(L.lpar_peer_gather_bytes(n, codec), fill=0) for _ in range(N)]
        self.flags = [Guarded(L.lpar_peer_flag_bytes(N, n), fill=0) for _ in range(N)]
        self.status = torch.zeros(8, dtype=torch.int32, device="cuda")
        self.epoch = 0

    def call(self, L, ins, outs):
        self.epoch += 1
        L.lpar_allreduce_peer([g.ptr() for g in ins], [g.ptr() for g in outs], [g.ptr() for g in self.mbox],
                              [g.ptr() for g in self.gath], [g.ptr() for g in self.flags], self.n, self.codec,
                              TIMEOUT_NS, self.status)
        torch.cuda.synchronize()
        assert self.status.tolist() == [0, 0, 0, 0, self.epoch, 0, 0, 0]   # the launch advanced the epoch
        for g in self.mbox + self.gath + self.flags:
            g.check()
        flags = [g.host().view(np.uint32) for g in self.flags]
        for f in flags:                                    # every flag of a non-empty chunk carries the epoch
            assert np.all((f == self.epoch) | (f == 0))


def inputs(N, n, seed):
    return [adversarial_bf16(n, seed + r) if r % 2 else random_bf16(n, seed + 50 + r, 2.0 ** (r - 3))
            for r in range(N)]


def check_exchange(L, b, xs, codec):
    """Mailbox slots and gathered wires against the oracle's wires."""
    N, n = len(xs), xs[0].size
    T = n // 2048
    tb = L.lpar_tile_bytes(codec)
    wires = [O.quantize(x, codec) for x in xs] if codec != "bf16" else [x.view(np.uint8) for x in xs]
    slot = -(-T // N)
    for j in range(N):
        t0, t1 = j * T // N, (j + 1) * T // N
        host = b.mbox[j].host()
        for s in range(N):
            got = host[s * slot * tb:(s * slot + t1 - t0) * tb]
            assert np.array_equal(got, wires[s][t0 * tb:t1 * tb]), ("mailbox", j, s)
    gathered = O.reduce(wires, 0, T, codec) if codec != "bf16" else None
    for r in range(N):
        if gathered is not None:
            assert np.array_equal(b.gath[r].host(), gathered), ("gathered", r)


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("tiles", [1, 9, 37])
def test_peer_matches_oracle(L, codec, N, tiles):
    n = tiles * 2048
    xs = inputs(N, n, 8100 + 10 * N + tiles)
    ins = [to_device(x) for x in xs]
    outs = [Guarded(2 * n, fill=0) for _ in range(N)]
    b = Bufs(L, N, n, codec)
    b.call(L, ins, outs)
    ref, used = O.allreduce(xs, codec)
    assert used == codec
    for o in outs + ins:
        o.check()
    for r, o in enumerate(outs):
        assert np.array_equal(host_u16(o), ref[0]), (codec, N, tiles, r)
    check_exchange(L, b, xs, codec)


@pytest.mark.parametrize("codec", CODECS)
def test_peer_repeated_calls_reuse_the_buffers_and_in_place(L, codec):
    """Epochs 1..4 on one set of buffers, new inputs every call; the last call
    in place (outputs = inputs)."""
    N, tiles = 3, 11
    n = tiles * 2048
    b = Bufs(L, N, n, codec)
    for k in range(4):
        xs = inputs(N, n, 8300 + 10 * k)
        ins = [to_device(x) for x in xs]
        outs = ins if k == 3 else [Guarded(2 * n, fill=0) for _ in range(N)]
        b.call(L, ins, outs)
        ref, _ = O.allreduce(xs, codec)
        for o in outs:
            o.check()
            assert np.array_equal(host_u16(o), ref[0]), (codec, k)


@pytest.mark.parametrize("codec", ["int4", "fp8", "bf16"])
def test_peer_calls_replayed_from_a_cuda_graph(L, codec):
    """The epoch lives in the status words, so one captured launch replayed
    five times (new inputs copied in before each replay) gives the oracle's
    result every time and advances the epoch by one per replay."""
    N, tiles = 4, 13
    n = tiles * 2048
    ins = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(N)]
    outs = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(N)]
    buf = L.PeerBuffers(N, n, codec)
    buf.allreduce(ins, outs)                              # warm-up outside the capture (epoch 1)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            buf.allreduce(ins, outs)
    torch.cuda.synchronize()
    for k in range(5):
        xs = inputs(N, n, 8900 + 10 * k)
        for d, x in zip(ins, xs):
            d.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        buf.check()
        assert buf.epoch() == 2 + k
        ref, _ = O.allreduce(xs, codec)
        for o in outs:
            assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), ref[0]), (codec, k)
    del graph


@pytest.mark.parametrize("case", range(24))
def test_peer_random_cases(L, case):
    """Seeded random cases over codec, N in 1..8, 1..700 tiles, in place or not,
    adversarial or scaled Gaussian inputs per rank; two calls on one set of
    buffers; every output bit for bit against the oracle."""
    rng = np.random.default_rng(8950 + case)
    codec = CODECS[rng.integers(len(CODECS))]
    N = int(rng.integers(1, 9))
    tiles = int(rng.integers(1, 701))
    n = tiles * 2048
    inplace = bool(rng.integers(2))
    b = Bufs(L, N, n, codec)
    for k in range(2):
        xs = [adversarial_bf16(n, int(rng.integers(1 << 30))) if rng.integers(2)
              else random_bf16(n, int(rng.integers(1 << 30)), float(2.0 ** rng.integers(-8, 9))) for _ in range(N)]
        ins = [to_device(x) for x in xs]
        outs = ins if inplace else [Guarded(2 * n, fill=0) for _ in range(N)]
        b.call(L, ins, outs)
        ref, _ = O.allreduce(xs, codec)
        for o in outs:
            o.check()
            assert np.array_equal(host_u16(o), ref[0]), (codec, N, tiles, inplace, k)


def chunks_per_shard(N, T):
    """The library's chunk count: chunks of about N T / 592 tiles (1 to 16, a
    multiple of 4 above 4), at most 1024 per shard."""
    ct = min(max(-(-(N * T) // 592), 1), 16)
    if ct > 4:
        ct = -(-ct // 4) * 4
    return min(max(-(-(-(-T // N)) // ct), 1), 1024)


def sampled(xs_dev, tiles):
    idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
    return idx, [x[idx].view(torch.int16).cpu().numpy().view(np.uint16) for x in xs_dev]


@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "mxfp4", "bf16"])
@pytest.mark.parametrize("N,T", [(2, 4099), (5, 5 * 3 * 1024 + 7), (8, 1024 * 8 + 2), (2, 2 * 16 * 1024 + 6)])
def test_peer_many_tile_chunks(L, codec, N, T):
    """Shards cut into many chunks of several tiles, ragged (the last case at
    the cap of 1024 chunks per shard); every chunk boundary of shard 0 and 1
    and 256 random tiles compared with the oracle, and the whole of rank 0's
    output with lpar_allreduce's."""
    n = T * 2048
    xs = [to_device(x) for x in inputs(N, n, 8400 + N)]
    outs = [Guarded(2 * n, fill=0) for _ in range(N)]
    b = Bufs(L, N, n, codec)
    b.call(L, xs, outs)
    P = chunks_per_shard(N, T)
    bounds = []
    for j in (0, 1):
        base, S = j * T // N, (j + 1) * T // N - j * T // N
        bounds += [base + c * S // P for c in range(P)] + [base + c * S // P - 1 for c in range(1, P + 1)]
    rng = np.random.default_rng(8500 + N)
    tiles = np.unique(np.concatenate([bounds, rng.choice(T, 256, replace=False), [T - 1]]))
    idx, sample_in = sampled([x.t.view(torch.bfloat16) for x in xs], tiles)
    ref, _ = O.allreduce(sample_in, codec)
    for o in outs:
        o.check()
        assert np.array_equal(o.t.view(torch.bfloat16)[idx].view(torch.int16).cpu().numpy().view(np.uint16), ref[0])
    ws = torch.empty(L.lpar_workspace_bytes(N, n, codec), dtype=torch.uint8, device="cuda")
    want = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    L.lpar_allreduce([x.ptr() for x in xs], n, codec, [want] + [o.ptr() for o in outs[1:]], ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(want.view(torch.int16), outs[0].t.view(torch.int16))


@pytest.mark.parametrize("name", ["large_int3_int4"])
def test_peer_full_size_sampled(L, name):
    """1 GiB per rank, N = 2 (the large workload), every codec of it: 1024
    seeded random tiles plus the first and last against the oracle."""
    w = W.WORKLOADS[name]
    xs = W.make_inputs(w, "cuda")
    T = w.n // 2048
    rng = np.random.default_rng(8600)
    tiles = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 1024, replace=False)]))
    idx, sample_in = sampled(xs, tiles)
    for codec in w.codecs:
        outs = [torch.empty_like(x) for x in xs]
        buf = L.PeerBuffers(w.N, w.n, codec)
        buf.allreduce(xs, outs)
        buf.check()
        ref, _ = O.allreduce(sample_in, codec)
        for o in outs:
            assert np.array_equal(o[idx].view(torch.int16).cpu().numpy().view(np.uint16), ref[0]), codec
        del outs, buf
    del xs
    torch.cuda.empty_cache()


def test_peer_wait_gives_up_on_a_rank_that_never_runs(L):
    """N = 2, the launch runs rank 0 only; rank 1's buffers are pinned host
    memory and nothing ever runs rank 1, so its flags are never raised.  Rank
    0's waits give up after the timeout (for rank 1's mailbox tiles, or for
    gathered tiles that never come), the status words say so, and the context
    still runs a normal call afterwards."""
    N, tiles, codec = 2, 6, "int4"
    n = tiles * 2048
    xs = inputs(N, n, 8700)
    x0 = to_device(xs[0])
    out0 = Guarded(2 * n, fill=0)
    mb0 = Guarded(L.lpar_peer_mailbox_bytes(N, n, codec), fill=0)
    ga0 = Guarded(L.lpar_peer_gather_bytes(n, codec), fill=0)
    fl0 = Guarded(L.lpar_peer_flag_bytes(N, n), fill=0)
    host = [torch.zeros(max(k, 16), dtype=torch.uint8, pin_memory=True)
            for k in (L.lpar_peer_mailbox_bytes(N, n, codec), L.lpar_peer_gather_bytes(n, codec),
                      L.lpar_peer_flag_bytes(N, n))]
    status = torch.zeros(8, dtype=torch.int32, device="cuda")
    timeout = 50_000_000                                  # 50 ms
    t0 = time.perf_counter()
    L.lpar_allreduce_peer([x0.ptr(), None], [out0.ptr(), None], [mb0.ptr(), host[0].data_ptr()],
                          [ga0.ptr(), host[1].data_ptr()], [fl0.ptr(), host[2].data_ptr()], n, codec, timeout,
                          status, rank0=0, ranks=1)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    w = status.tolist()
    P = chunks_per_shard(N, tiles)
    # the first wait to give up is rank 0's, for source 1's mailbox tiles (phase 1: flags
    # [P, 2P)) or for gathered tiles that a blocked owner never sent (phase 2: flags [2P, 4P));
    # which one depends on which CTA started waiting first
    assert w[0] == 1 and w[2] == 0, w
    assert (w[1] == 1 and P <= w[3] < 2 * P) or (w[1] == 2 and 2 * P <= w[3] < 4 * P), w
    assert w[4:] == [1, 0, 0, 0], w                        # epoch 1 done, every CTA accounted for
    assert elapsed < 5.0, elapsed
    for g in (out0, mb0, ga0, fl0):
        g.check()
    # rank 0's phase A did reach rank 1: its tiles of shard 1 are in rank 1's mailbox, slot 0
    wire0 = O.quantize(xs[0], codec)
    tb, t1 = L.lpar_tile_bytes(codec), tiles // N
    assert np.array_equal(host[0][:(tiles - t1) * tb].numpy(), wire0[t1 * tb:])
    assert np.all(host[2].numpy().view(np.uint32)[:P] == 1)
    # a launch that finds the status set does nothing
    out1 = Guarded(2 * n, fill=0x33)
    L.lpar_allreduce_peer([x0.ptr(), None], [out1.ptr(), None], [mb0.ptr(), host[0].data_ptr()],
                          [ga0.ptr(), host[1].data_ptr()], [fl0.ptr(), host[2].data_ptr()], n, codec, timeout,
                          status, rank0=0, ranks=1)
    torch.cuda.synchronize()
    assert np.all(out1.host() == 0x33)
    assert status.tolist()[:5] == w[:4] + [2]
    # the context is intact: a normal all-reduce of both ranks
    out = L.allreduce_peer([torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in xs], codec)
    torch.cuda.synchronize()
    ref, _ = O.allreduce(xs, codec)
    for o in out:
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), ref[0])


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,d,tiles", [(2, 0, 9), (2, 1, 40), (3, 1, 37), (3, 2, 100)])
def test_peer_one_rank_against_host_played_peers(L, codec, N, d, tiles):
    """The form one rank per GPU runs (ranks = 1, system-scope flags, wire tiles
    staged in shared memory and stored into another rank's memory), with the
    other ranks played by the host: their buffers are pinned host memory, and
    before the launch the host writes into rank d's buffers everything they
    would have sent -- their stage-1 tiles of shard d (the oracle's wires), the
    reduced shards they own (the oracle's reduction) -- and raises the matching
    flags.  Every wait of the launch is therefore already satisfied (nothing
    else runs).  Rank d's output, and what its launch stored into the host
    ranks' mailboxes, gathered wires and flags, must match the oracle."""
    n = tiles * 2048
    T, tb = tiles, L.lpar_tile_bytes(codec)
    xs = inputs(N, n, 8800 + 10 * N + d)
    P = chunks_per_shard(N, T)
    slot = -(-T // N)
    shard = [(j * T // N, (j + 1) * T // N) for j in range(N)]
    if codec == "bf16":
        wires = [x.view(np.uint8) for x in xs]
        ref, _ = O.allreduce(xs, codec)
        gathered = ref[0].view(np.uint8)
    else:
        wires = [O.quantize(x, codec) for x in xs]
        gathered = O.reduce(wires, 0, T, codec)
        ref, _ = O.allreduce(xs, codec)
    mb_bytes, ga_bytes, fl_bytes = (L.lpar_peer_mailbox_bytes(N, n, codec), L.lpar_peer_gather_bytes(n, codec),
                                    L.lpar_peer_flag_bytes(N, n))
    assert fl_bytes == 2 * N * P * 4
    # rank d: device buffers holding what the host-played ranks sent
    mb = np.zeros(mb_bytes, np.uint8)
    ga = np.zeros(ga_bytes, np.uint8)
    fl = np.zeros(2 * N * P, np.uint32)
    t0, t1 = shard[d]
    for h in range(N):
        if h == d:
            continue
        mb[h * slot * tb:(h * slot + t1 - t0) * tb] = wires[h][t0 * tb:t1 * tb]
        fl[h * P:(h + 1) * P] = 1                                  # source h's mailbox chunks of shard d
        a0, a1 = shard[h]
        ga[a0 * tb:a1 * tb] = gathered[a0 * tb:a1 * tb]            # shard h, reduced by its owner
        fl[N * P + h * P:N * P + (h + 1) * P] = 1
    dev = [Guarded(mb_bytes, fill=0), Guarded(ga_bytes, fill=0), Guarded(fl_bytes, fill=0)]
    for g, arr in zip(dev, (mb, ga, fl.view(np.uint8))):
        g.t.copy_(torch.from_numpy(arr))
    host = {h: [torch.zeros(k, dtype=torch.uint8, pin_memory=True) for k in (mb_bytes, ga_bytes, fl_bytes)]
            for h in range(N) if h != d}
    x_d = to_device(xs[d])
    out_d = Guarded(2 * n, fill=0)
    status = torch.zeros(8, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    ptrs = lambda k: [dev[k].ptr() if r == d else host[r][k].data_ptr() for r in range(N)]
    L.lpar_allreduce_peer([x_d.ptr() if r == d else None for r in range(N)],
                          [out_d.ptr() if r == d else None for r in range(N)], ptrs(0), ptrs(1), ptrs(2), n, codec,
                          TIMEOUT_NS, status, rank0=d, ranks=1)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0, 0, 0, 1, 0, 0, 0]
    for g in dev + [out_d, x_d]:
        g.check()
    assert np.array_equal(host_u16(out_d), ref[0]), (codec, N, d)
    for h, (hmb, hga, hfl) in host.items():
        a0, a1 = shard[h]
        assert np.array_equal(hmb.numpy()[d * slot * tb:(d * slot + a1 - a0) * tb], wires[d][a0 * tb:a1 * tb])
        assert np.array_equal(hga.numpy()[t0 * tb:t1 * tb], gathered[t0 * tb:t1 * tb])   # rank d's reduced shard
        f = hfl.numpy().view(np.uint32)
        for c in range(P):
            lo_h, hi_h = a0 + c * (a1 - a0) // P, a0 + (c + 1) * (a1 - a0) // P
            assert f[d * P + c] == (1 if hi_h > lo_h else 0), ("mailbox flag", h, c)
            lo_d, hi_d = t0 + c * (t1 - t0) // P, t0 + (c + 1) * (t1 - t0) // P
            assert f[N * P + d * P + c] == (1 if hi_d > lo_d else 0), ("gathered flag", h, c)
        untouched = np.ones(mb_bytes, bool)
        untouched[d * slot * tb:(d * slot + a1 - a0) * tb] = False
        assert not hmb.numpy()[untouched].any()                      # nothing outside rank d's slot


def test_peer_refuses_an_absent_rank_on_this_device(L):
    """A rank outside the launch whose buffers are this GPU's memory would have
    to be a second launch on the same GPU waiting on this one: refused before
    anything is launched."""
    N, n, codec = 2, 2048 * 4, "int4"
    bufs = [torch.zeros(max(k, 16), dtype=torch.uint8, device="cuda")
            for k in (L.lpar_peer_mailbox_bytes(N, n, codec), L.lpar_peer_gather_bytes(n, codec),
                      L.lpar_peer_flag_bytes(N, n))] * 2
    x = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(8, dtype=torch.int32, device="cuda")
    with pytest.raises(L.LparError) as e:
        L.lpar_allreduce_peer([x, None], [x, None], [bufs[0], bufs[3]], [bufs[1], bufs[4]], [bufs[2], bufs[5]], n,
                              codec, TIMEOUT_NS, status, rank0=0, ranks=1)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert status.tolist() == [0] * 8
    # host memory the GPU cannot reach (pageable) is refused the same way
    pageable = [np.zeros(max(k, 16), np.uint8) for k in (L.lpar_peer_mailbox_bytes(N, n, codec),
                                                          L.lpar_peer_gather_bytes(n, codec),
                                                          L.lpar_peer_flag_bytes(N, n))]
    with pytest.raises(L.LparError) as e:
        L.lpar_allreduce_peer([x, None], [x, None], [bufs[0], pageable[0].ctypes.data],
                              [bufs[1], pageable[1].ctypes.data], [bufs[2], pageable[2].ctypes.data], n, codec,
                              TIMEOUT_NS, status, rank0=0, ranks=1)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert status.tolist() == [0] * 8


# ---------------------------------------------------------------------------
# CUDA IPC across processes on the one GPU.
# ---------------------------------------------------------------------------
class _Raw:
    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False), "version": 3}


def _layout(L, N, n, codec):
    """Byte offsets of input, output, mailbox, gathered wire and flags in one
    exported region (each 256-byte aligned)."""
    sizes = [2 * n, 2 * n, L.lpar_peer_mailbox_bytes(N, n, codec), L.lpar_peer_gather_bytes(n, codec),
             L.lpar_peer_flag_bytes(N, n)]
    offs, o = [], 0
    for s in sizes:
        offs.append(o)
        o += -(-s // 256) * 256
    return offs, o


def _ipc_worker(rank, world, port, n, codec, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_precision_all_b200 import lpar as L
        offs, total = _layout(L, world, n, codec)
        region = L.lpar_peer_alloc(total)
        view = torch.as_tensor(_Raw(region, total), device="cuda")
        x = inputs(world, n, 8800)[rank]
        view[offs[0]:offs[0] + 2 * n].copy_(torch.from_numpy(x.view(np.uint8)))
        torch.cuda.synchronize()
        handles = [None] * world
        dist.all_gather_object(handles, L.lpar_peer_export(region))
        if rank == 0:
            bases = [region] + [L.lpar_peer_import(h) for h in handles[1:]]
            status = torch.zeros(8, dtype=torch.int32, device="cuda")
            ptr = lambda k: [b + offs[k] for b in bases]
            L.lpar_allreduce_peer(ptr(0), ptr(1), ptr(2), ptr(3), ptr(4), n, codec, TIMEOUT_NS, status)
            torch.cuda.synchronize()
            st = status.tolist()
            for b in bases[1:]:
                L.lpar_peer_close(b)
        else:
            st = None
        dist.barrier()
        out = view[offs[1]:offs[1] + 2 * n].cpu().numpy().copy()
        dist.barrier()
        L.lpar_peer_free(region)
        q.put((rank, out, st))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,tiles,codec", [(2, 7, "int3"), (3, 10, "fp8")])
def test_peer_buffers_shared_by_ipc(world, tiles, codec):
    import torch.multiprocessing as mp
    n = tiles * 2048
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, n, codec, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, out, st = q.get(timeout=300)
        got[r] = (out, st)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert got[0][1] == [0, 0, 0, 0, 1, 0, 0, 0]
    ref, _ = O.allreduce(inputs(world, n, 8800), codec)
    for r in range(world):
        assert np.array_equal(got[r][0].view(np.uint16), ref[0]), r


def _shared_gpu_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_precision_all_b200.distributed import PeerAllreduce
        try:
            PeerAllreduce()
            q.put((rank, None))
        except ValueError as e:
            q.put((rank, str(e)))
    finally:
        dist.destroy_process_group()


def test_peer_allreduce_refuses_ranks_that_share_a_gpu():
    """Two processes on the one GPU: PeerAllreduce's construction sees the same
    GPU UUID twice and raises on both ranks before anything is allocated."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shared_gpu_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        assert got[r] is not None and "share GPU" in got[r], got
