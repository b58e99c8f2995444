"""The compressed all-reduce across processes, one GPU per rank.

This is the two-shot schedule of the single-GPU emulation with the exchange
steps made real ("RCCLX: Innovating GPU communications on AMD platforms",
Direct Data Access: the tree all-reduce is a reduce-scatter followed by an
all-gather; Low-Precision Collectives: the quantised wire is what crosses the
links, compute stays in FP32):

  1. every rank quantises its message into its wire (``lpar_quantize``);
  2. all-to-all of wire shards: rank j receives shard j (tiles
     [jT/N, (j+1)T/N), the same floor partition as the emulation) of every
     rank's wire, in rank order;
  3. rank j reduces its shard from the N received wires and requantises it
     (``lpar_reduce``: FP32 sum in ascending rank order from +0.0f), straight
     into its slot of the all-gather buffer;
  4. all-gather of the requantised shards into one buffer (slots padded to the
     largest shard);
  5. every rank decodes each shard from its slot into its place of the output
     (``lpar_decode``): no concatenation or other copy of the gathered wire.

The result is bit-identical to ``lpar_allreduce`` on the N messages in one GPU.
The exchanges use ``torch.distributed`` collectives on the wire bytes (NCCL on
GPUs); the arithmetic runs in the library's kernels.  The stage functions are
an argument so that the host orchestration can be exercised on its own.
"""
from dataclasses import dataclass
from typing import Callable, List, Optional

import torch
import torch.distributed as dist

from . import lpar as L

TILE_ELEMS = L.TILE_ELEMS


@dataclass
class Stages:
    """quantize(x, codec) -> wire; reduce(wires, tiles, codec, out) writes the
    reduced wire of `tiles` tiles into `out`; decode(wire, n, codec, out) writes
    n BF16 values into `out`; tile_bytes(codec)."""
    quantize: Callable
    reduce: Callable
    decode: Callable
    tile_bytes: Callable


def cuda_stages(stream: Optional[torch.cuda.Stream] = None) -> Stages:
    """The library's kernels on the current device (the product path)."""
    def quantize(x, codec):
        wire = torch.empty(L.lpar_wire_bytes(codec, x.numel()), dtype=torch.uint8, device=x.device)
        L.lpar_quantize(x, x.numel(), codec, wire, stream)
        return wire

    def reduce(wires, tiles, codec, out):
        if tiles:
            L.lpar_reduce(list(wires), 0, tiles, codec, out, stream)

    def decode(wire, n, codec, out):
        L.lpar_decode(wire, n, codec, out, stream)

    return Stages(quantize, reduce, decode, L.lpar_tile_bytes)


def shard_tiles(N: int, T: int) -> List[tuple]:
    """Tile range [t0, t1) of shard j, j = 0..N-1 (floor partition)."""
    return [(j * T // N, (j + 1) * T // N) for j in range(N)]


class DistributedAllreduce:
    """All-reduce of one BF16 tensor per process across a process group."""

    def __init__(self, group=None, stages: Optional[Stages] = None):
        self.group = group
        self.N = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.stages = stages if stages is not None else cuda_stages()

    def allreduce(self, x: torch.Tensor, codec: str, min_quant_bytes: int = 0,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
        n = x.numel()
        if n % TILE_ELEMS:
            raise ValueError("the message must be a whole number of 2048-element tiles")
        if codec != "bf16" and 2 * n < min_quant_bytes:
            codec = "bf16"                                  # the threshold on the per-rank message
        N, me, st = self.N, self.rank, self.stages
        T = n // TILE_ELEMS
        tb = st.tile_bytes(codec)
        shards = shard_tiles(N, T)
        wire = st.quantize(x, codec)                        # 1. stage 1
        # 2. all-to-all: my shard's tiles from every rank, in rank order
        send_sizes = [(t1 - t0) * tb for t0, t1 in shards]
        my_tiles = shards[me][1] - shards[me][0]
        recv = torch.empty(N * my_tiles * tb, dtype=torch.uint8, device=wire.device)
        dist.all_to_all_single(recv, wire, output_split_sizes=[my_tiles * tb] * N,
                               input_split_sizes=send_sizes, group=self.group)
        received = [recv[r * my_tiles * tb:(r + 1) * my_tiles * tb] for r in range(N)]
        # 3. stage 2 of my shard, straight into my slot of the all-gather (padded
        #    to the largest shard; the padding is never decoded)
        width = max(t1 - t0 for t0, t1 in shards) * tb
        send = torch.empty(width, dtype=torch.uint8, device=wire.device)
        st.reduce(received, my_tiles, codec, send[:my_tiles * tb])
        # 4. all-gather of the shards into one buffer, rank j's slot at j * width
        gathered = torch.empty(N * width, dtype=torch.uint8, device=wire.device)
        dist.all_gather(list(gathered.view(N, width).unbind(0)), send, group=self.group)
        # 5. stage 3: each shard decoded from its slot into its place of the output
        if out is None:
            out = torch.empty(n, dtype=torch.bfloat16, device=x.device)
        for j, (t0, t1) in enumerate(shards):
            if t1 > t0:
                st.decode(gathered[j * width:j * width + (t1 - t0) * tb], (t1 - t0) * TILE_ELEMS, codec,
                          out[t0 * TILE_ELEMS:t1 * TILE_ELEMS])
        return out
