"""The compressed all-reduce across processes, one GPU per rank.

This is the two-shot schedule of the single-GPU emulation with the exchange
steps made real ("RCCLX: Innovating GPU communications on AMD platforms",
Direct Data Access: the tree all-reduce is a reduce-scatter followed by an
all-gather; Low-Precision Collectives: the quantised wire is what crosses the
links, compute stays in FP32).  For each chunk of the message (a range of
whole tiles; tiles are independent, so chunking changes no result):

  1. every rank quantises its chunk into its wire (``lpar_quantize``);
  2. all-to-all of wire shards: rank j receives shard j of the chunk (tiles
     [jT/N, (j+1)T/N) of its T tiles, the emulation's floor partition) of
     every rank's wire, in rank order;
  3. rank j reduces its shard from the N received wires and requantises it
     (``lpar_reduce``: FP32 sum in ascending rank order from +0.0f) into its
     send slot;
  4. all-gather of the requantised shards into one buffer (slots padded to
     the largest shard);
  5. every rank decodes each shard from its slot into its place of the output
     (``lpar_decode``): no concatenation or other copy of the gathered wire.

The exchanges of chunk k are issued asynchronously, so with NCCL they run on
its own stream while the kernels of chunk k + 1 run on the compute stream:
the all-to-all of chunk k overlaps the quantisation of chunk k + 1, and the
all-gather of chunk k the reduction of chunk k + 1.

The result is bit-identical to ``lpar_allreduce`` on the N messages in one
GPU.  ``PeerAllreduce`` is the same all-reduce with the exchanges folded into
the library's peer-memory kernel (``lpar_allreduce_peer``): one launch per
rank stores its wire tiles straight into the owners' memory and the reduced
shard into every rank's memory, over CUDA IPC mappings, with no separate
collective on the data path.  The exchanges use ``torch.distributed`` collectives on the wire bytes;
the arithmetic runs in the library's kernels.  Buffers are allocated once per
(message size, codec, device) and reused by later calls.  With a process group
that cannot move device memory (gloo), the wire bytes travel through host
copies of the exchange buffers.  The stage functions are an argument so that
the host orchestration can also be exercised with other implementations.
"""
from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import lpar as L

TILE_ELEMS = L.TILE_ELEMS


@dataclass
class Stages:
    """quantize(x, codec, wire) writes x's wire into `wire`; reduce(wires,
    tiles, codec, out) writes the reduced wire of `tiles` tiles into `out`;
    decode(wire, n, codec, out) writes n BF16 values into `out`;
    tile_bytes(codec)."""
    quantize: Callable
    reduce: Callable
    decode: Callable
    tile_bytes: Callable


def cuda_stages(stream=None) -> Stages:
    """The library's kernels on the current device (the product path)."""
    def quantize(x, codec, wire):
        L.lpar_quantize(x, x.numel(), codec, wire, stream)

    def reduce(wires, tiles, codec, out):
        if tiles:
            L.lpar_reduce(list(wires), 0, tiles, codec, out, stream)

    def decode(wire, n, codec, out):
        L.lpar_decode(wire, n, codec, out, stream)

    return Stages(quantize, reduce, decode, L.lpar_tile_bytes)


def shard_tiles(N: int, T: int) -> List[Tuple[int, int]]:
    """Tile range [t0, t1) of shard j, j = 0..N-1 (floor partition)."""
    return [(j * T // N, (j + 1) * T // N) for j in range(N)]


def chunk_tiles(T: int, chunks: int) -> List[Tuple[int, int]]:
    """The message's tiles split into at most `chunks` contiguous ranges."""
    k = max(1, min(chunks, T))
    return [(c * T // k, (c + 1) * T // k) for c in range(k)]


class _Buffers:
    """Exchange buffers of one (tiles per chunk, codec, device): the rank's
    wire, the received shards, the send slot and the gathered slots, one set per
    chunk in flight; plus host copies when the group moves host memory only."""

    def __init__(self, N, me, chunk_ranges, tb, device, host):
        self.plans = []
        for t0, t1 in chunk_ranges:
            T = t1 - t0
            shards = shard_tiles(N, T)
            mine = shards[me][1] - shards[me][0]
            width = max(b - a for a, b in shards) * tb
            plan = {
                "T": T, "shards": shards, "mine": mine, "width": width,
                "wire": torch.empty(T * tb, dtype=torch.uint8, device=device),
                "recv": torch.empty(N * mine * tb, dtype=torch.uint8, device=device),
                "send": torch.empty(width, dtype=torch.uint8, device=device),
                "gathered": torch.empty(N * width, dtype=torch.uint8, device=device),
            }
            if host:
                for k in ("wire", "recv", "send", "gathered"):
                    plan["h_" + k] = torch.empty(plan[k].numel(), dtype=torch.uint8,
                                                 pin_memory=torch.cuda.is_available() and device.type == "cuda")
            self.plans.append(plan)


class DistributedAllreduce:
    """All-reduce of one BF16 tensor per process across a process group.

    chunks: the message is processed in up to this many tile ranges, so that
    the exchange of one overlaps the kernels of the next.  exchange_on_host:
    route the wire bytes through host buffers (default: when the group's
    backend is gloo and the data lives on a GPU)."""

    def __init__(self, group=None, stages: Optional[Stages] = None, chunks: int = 1,
                 exchange_on_host: Optional[bool] = None):
        self.group = group
        self.N = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.stages = stages if stages is not None else cuda_stages()
        self.chunks = max(1, int(chunks))
        self.exchange_on_host = exchange_on_host
        self._cache: Dict[tuple, _Buffers] = {}

    def _host(self, device) -> bool:
        if self.exchange_on_host is not None:
            return bool(self.exchange_on_host)
        return device.type == "cuda" and dist.get_backend(self.group) == "gloo"

    def buffers(self, n: int, codec: str, device) -> _Buffers:
        key = (n, codec, str(device))
        b = self._cache.get(key)
        if b is None:
            T = n // TILE_ELEMS
            b = _Buffers(self.N, self.rank, chunk_tiles(T, self.chunks), self.stages.tile_bytes(codec), device,
                         self._host(device))
            self._cache[key] = b
        return b

    def release(self):
        """Drop the cached exchange buffers."""
        self._cache.clear()

    # -- the two exchanges, on device buffers or through their host copies ----
    def _all_to_all(self, p, tb, host):
        N, mine = self.N, p["mine"]
        in_splits = [(t1 - t0) * tb for t0, t1 in p["shards"]]
        out_splits = [mine * tb] * N
        if host:
            p["h_wire"].copy_(p["wire"])
            dist.all_to_all_single(p["h_recv"], p["h_wire"], output_split_sizes=out_splits,
                                   input_split_sizes=in_splits, group=self.group)
            p["recv"].copy_(p["h_recv"])
            return None
        return dist.all_to_all_single(p["recv"], p["wire"], output_split_sizes=out_splits,
                                      input_split_sizes=in_splits, group=self.group, async_op=True)

    def _all_gather(self, p, host):
        if host:
            p["h_send"].copy_(p["send"])
            dist.all_gather_into_tensor(p["h_gathered"], p["h_send"], group=self.group)
            p["gathered"].copy_(p["h_gathered"])
            return None
        return dist.all_gather_into_tensor(p["gathered"], p["send"], group=self.group, async_op=True)

    def allreduce(self, x: torch.Tensor, codec: str, min_quant_bytes: int = 0,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
        n = x.numel()
        if n % TILE_ELEMS:
            raise ValueError("the message must be a whole number of 2048-element tiles")
        if codec != "bf16" and 2 * n < min_quant_bytes:
            codec = "bf16"                                  # the threshold on the per-rank message
        if out is None:
            out = torch.empty(n, dtype=torch.bfloat16, device=x.device)
        if n == 0:
            return out
        st, tb = self.stages, self.stages.tile_bytes(codec)
        bufs = self.buffers(n, codec, x.device)
        host = self._host(x.device)
        ranges = chunk_tiles(n // TILE_ELEMS, self.chunks)
        a2a = []
        for (t0, t1), p in zip(ranges, bufs.plans):         # 1. stage 1, then 2. its all-to-all
            st.quantize(x[t0 * TILE_ELEMS:t1 * TILE_ELEMS], codec, p["wire"])
            a2a.append(self._all_to_all(p, tb, host))
        ag = []
        for h, p in zip(a2a, bufs.plans):                    # 3. stage 2 of my shard, 4. all-gather
            if h is not None:
                h.wait()
            mine = p["mine"]
            received = [p["recv"][r * mine * tb:(r + 1) * mine * tb] for r in range(self.N)]
            st.reduce(received, mine, codec, p["send"][:mine * tb])
            ag.append(self._all_gather(p, host))
        for (t0, t1), h, p in zip(ranges, ag, bufs.plans):   # 5. stage 3 of every shard
            if h is not None:
                h.wait()
            w = p["width"]
            for j, (s0, s1) in enumerate(p["shards"]):
                if s1 > s0:
                    a, b = (t0 + s0) * TILE_ELEMS, (t0 + s1) * TILE_ELEMS
                    st.decode(p["gathered"][j * w:j * w + (s1 - s0) * tb], b - a, codec, out[a:b])
        return out


# ---------------------------------------------------------------------------
# The peer-memory form: one kernel launch per rank, exchanges by stores into
# the other ranks' memory.
# ---------------------------------------------------------------------------
@dataclass
class PeerOps:
    """The library calls PeerAllreduce makes: alloc(nbytes) -> address (zeroed,
    exportable), free(addr), export(addr) -> handle bytes, import_(handle) ->
    address, close(addr), mailbox_bytes(N, n, codec), gather_bytes(n, codec),
    flag_bytes(N, n), and run(inputs, outputs, mailboxes, gathered, flags, n,
    codec, timeout_ns, status, rank0, ranks) for lpar_allreduce_peer."""
    alloc: Callable
    free: Callable
    export: Callable
    import_: Callable
    close: Callable
    mailbox_bytes: Callable
    gather_bytes: Callable
    flag_bytes: Callable
    run: Callable


def cuda_peer_ops() -> PeerOps:
    """The library's calls (the product path)."""
    return PeerOps(L.lpar_peer_alloc, L.lpar_peer_free, L.lpar_peer_export, L.lpar_peer_import, L.lpar_peer_close,
                   L.lpar_peer_mailbox_bytes, L.lpar_peer_gather_bytes, L.lpar_peer_flag_bytes,
                   lambda *a, **k: L.lpar_allreduce_peer(*a, **k))


def _align(x, a=256):
    return -(-x // a) * a


class _PeerRegion:
    """One rank's exportable region for one (n, codec) -- mailbox, gathered
    wire, flags -- the addresses of every rank's region in this process, and
    the status words of the calls on it (which carry their epoch)."""

    def __init__(self, ops, group, N, me, n, codec, device):
        self.ops = ops
        sizes = [ops.mailbox_bytes(N, n, codec), ops.gather_bytes(n, codec), ops.flag_bytes(N, n)]
        self.offsets = [0, _align(sizes[0]), _align(sizes[0]) + _align(sizes[1])]
        self.local = ops.alloc(self.offsets[2] + _align(sizes[2]))
        handles = [None] * N
        dist.all_gather_object(handles, ops.export(self.local), group=group)
        self.bases = [self.local if r == me else ops.import_(handles[r]) for r in range(N)]
        self.me = me
        self.status = torch.zeros(L.LPAR_PEER_STATUS_WORDS, dtype=torch.int32, device=device)

    def pointers(self, k):
        return [b + self.offsets[k] for b in self.bases]

    def release(self, group):
        for r, b in enumerate(self.bases):
            if r != self.me:
                self.ops.close(b)
        dist.barrier(group=group)                          # nobody maps our region any more
        self.ops.free(self.local)


class PeerAllreduce:
    """All-reduce of one BF16 tensor per process, one GPU per process, by the
    peer-memory kernel.  Each rank allocates an exportable region per (message
    size, codec) on first use; the regions' handles are exchanged over the
    process group and mapped in every process.  A call is one launch on this
    rank's GPU that runs this rank only; every rank must make the same calls in
    the same order (the calls on a region are counted by its epoch).  The ranks' GPUs
    must be distinct: construction (a collective call) compares the ranks'
    GPU UUIDs and raises ValueError when two ranks share a GPU.  `check()`
    synchronises and raises when a wait for another rank gave up (after
    timeout_ns without progress)."""

    def __init__(self, group=None, ops: Optional[PeerOps] = None, timeout_ns: int = 2_000_000_000,
                 device=None):
        self.group = group
        self.N = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.ops = ops if ops is not None else cuda_peer_ops()
        self.timeout_ns = int(timeout_ns)
        self.device = device if device is not None else (torch.device("cuda", torch.cuda.current_device())
                                                         if torch.cuda.is_available() else torch.device("cpu"))
        self._regions: Dict[tuple, _PeerRegion] = {}
        if self.device.type == "cuda":
            uuids = [None] * self.N
            dist.all_gather_object(uuids, str(torch.cuda.get_device_properties(self.device).uuid), group=group)
            for r in range(self.N):
                if uuids.index(uuids[r]) != r:
                    raise ValueError("PeerAllreduce needs one GPU per rank: ranks %d and %d share GPU %s"
                                     % (uuids.index(uuids[r]), r, uuids[r]))

    def region(self, n: int, codec: str) -> _PeerRegion:
        key = (n, codec)
        reg = self._regions.get(key)
        if reg is None:
            reg = _PeerRegion(self.ops, self.group, self.N, self.rank, n, codec, self.device)
            self._regions[key] = reg
        return reg

    def allreduce(self, x: torch.Tensor, codec: str, min_quant_bytes: int = 0,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
        n = x.numel()
        if n % TILE_ELEMS:
            raise ValueError("the message must be a whole number of 2048-element tiles")
        if codec != "bf16" and 2 * n < min_quant_bytes:
            codec = "bf16"
        if out is None:
            out = torch.empty(n, dtype=torch.bfloat16, device=x.device)
        if n == 0:
            return out
        reg = self.region(n, codec)
        ins = [x if r == self.rank else None for r in range(self.N)]
        outs = [out if r == self.rank else None for r in range(self.N)]
        self.ops.run(ins, outs, reg.pointers(0), reg.pointers(1), reg.pointers(2), n, codec, self.timeout_ns,
                     reg.status, rank0=self.rank, ranks=1)
        return out

    def check(self):
        """Synchronise and raise PeerTimeout if a wait of any call gave up."""
        for key in sorted(self._regions):
            w = [int(v) for v in self._regions[key].status.cpu()]
            if w[0]:
                raise L.PeerTimeout("rank %d: a wait gave up (phase %d, waiting rank %d, flag %d)"
                                    % (self.rank, w[1], w[2], w[3]))

    def epochs(self):
        """{(n, codec): epoch of the last call} (synchronises)."""
        return {key: int(reg.status[4]) & 0xFFFFFFFF for key, reg in self._regions.items()}

    def release(self):
        """Unmap the peers' regions and free this rank's (collective: every rank
        calls it; no call may be in flight)."""
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        for key in sorted(self._regions):
            self._regions[key].release(self.group)
        self._regions.clear()
