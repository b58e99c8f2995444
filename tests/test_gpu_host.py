"""lpar_allreduce_host on the GPU against the CPU oracle, bit for bit (needs a
B200): messages in host memory, reduced chunk by chunk through device staging
with the copies and kernels overlapped.  The result must equal the oracle's
all-reduce of the whole message: several chunks, a ragged last chunk, more
chunks than staging slots, in place on the host, pageable host memory, the
threshold decided on the whole message, and every schedule.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.test_gpu_parity import adversarial_bf16

pytestmark = pytest.mark.gpu

CODECS = ("int4", "int3", "fp8", "mxfp4", "bf16")


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


def host_tensor(bits, pinned=True):
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.pin_memory() if pinned else t


def run(L, xs, codec, chunk, min_quant_bytes=0, schedule="auto", inplace=False, pinned=True):
    N, n = len(xs), xs[0].size
    hin = [host_tensor(x, pinned) for x in xs]
    hout = hin if inplace else [host_tensor(np.zeros(n, np.uint16), pinned) for _ in range(N)]
    eff = L.lpar_effective_codec(n, codec, min_quant_bytes)
    c = min(chunk, n)
    dev = torch.empty(L.lpar_host_staging_bytes(N, c, eff), dtype=torch.uint8, device="cuda")
    L.lpar_allreduce_host(hin, n, codec, hout, chunk, dev, dev.numel(), min_quant_bytes, schedule)
    torch.cuda.current_stream().synchronize()
    return [o.view(torch.int16).numpy().view(np.uint16) for o in hout], eff


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles,chunk_tiles", [(1, 5, 2), (2, 11, 4), (3, 9, 2), (8, 7, 3)])
def test_matches_oracle_whole_message(L, codec, N, tiles, chunk_tiles):
    n = tiles * 2048
    xs = [adversarial_bf16(n, 3100 + 10 * N + r) for r in range(N)]
    outs, eff = run(L, xs, codec, chunk_tiles * 2048)
    ref, used = O.allreduce(xs, codec)
    assert eff == used == codec
    for o in outs:
        assert np.array_equal(o, ref[0]), (codec, N)


@pytest.mark.parametrize("codec", ["int3", "fp8"])
def test_in_place_on_the_host(L, codec):
    xs = [adversarial_bf16(2048 * 10, 3200 + r) for r in range(2)]
    outs, _ = run(L, xs, codec, 2048 * 3, inplace=True)
    ref, _ = O.allreduce(xs, codec)
    for o in outs:
        assert np.array_equal(o, ref[0])


def test_pageable_host_memory(L):
    xs = [adversarial_bf16(2048 * 6, 3300 + r) for r in range(3)]
    outs, _ = run(L, xs, "int4", 2048 * 2, pinned=False)
    ref, _ = O.allreduce(xs, "int4")
    for o in outs:
        assert np.array_equal(o, ref[0])


def test_threshold_on_the_whole_message(L):
    n = 2048 * 8
    xs = [adversarial_bf16(n, 3400 + r) for r in range(2)]
    thr = 2 * n                                       # the whole message qualifies, a chunk would not
    outs, eff = run(L, xs, "int3", 2048 * 2, min_quant_bytes=thr)
    ref, used = O.allreduce(xs, "int3", thr)
    assert eff == used == "int3"
    assert np.array_equal(outs[0], ref[0])
    outs, eff = run(L, xs, "int3", 2048 * 2, min_quant_bytes=thr + 2)
    ref, used = O.allreduce(xs, "int3", thr + 2)
    assert eff == used == "bf16"
    assert np.array_equal(outs[0], ref[0])


@pytest.mark.parametrize("schedule", ["fused", "three_stage", "single_pass"])
def test_every_schedule_gives_the_same_bits(L, schedule):
    xs = [adversarial_bf16(2048 * 9, 3500 + r) for r in range(4)]
    outs, _ = run(L, xs, "mxfp4", 2048 * 4, schedule=schedule)
    ref, _ = O.allreduce(xs, "mxfp4")
    for o in outs:
        assert np.array_equal(o, ref[0])


def test_one_shot_schedule(L):
    xs = [adversarial_bf16(2048 * 9, 3600 + r) for r in range(3)]
    outs, _ = run(L, xs, "int4", 2048 * 2, schedule="one_shot")
    ref, _ = O.allreduce_oneshot(xs, "int4")
    for o in outs:
        assert np.array_equal(o, ref[0])


def test_helper_and_stream_order(L):
    """The Python helper allocates pinned outputs and staging; later work on the
    caller's stream sees the results in host memory."""
    n = 2048 * 64
    xs = [adversarial_bf16(n, 3700 + r) for r in range(2)]
    hin = [host_tensor(x) for x in xs]
    outs = L.allreduce_host(hin, "int3", chunk=2048 * 8)
    flag = torch.zeros(1, device="cuda")
    flag += 1                                          # later work on the same stream
    torch.cuda.current_stream().synchronize()
    ref, _ = O.allreduce(xs, "int3")
    for o in outs:
        assert o.is_pinned()
        assert np.array_equal(o.view(torch.int16).numpy().view(np.uint16), ref[0])


# ---- binary32 messages: lpar_allreduce_f32_host ------------------------------------
@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles,chunk_tiles", [(2, 7, 2), (8, 5, 3)])
def test_f32_host_matches_oracle(L, codec, N, tiles, chunk_tiles):
    from tests.test_gpu_f32 import adversarial_f32
    n = tiles * 2048
    xs = [adversarial_f32(n, 3800 + 10 * N + r) for r in range(N)]
    hin = [torch.from_numpy(x.copy()).pin_memory() for x in xs]
    hout = [torch.zeros(n, dtype=torch.float32).pin_memory() for _ in range(N)]
    eff = L.lpar_effective_codec(2 * n, codec, 0)
    c = chunk_tiles * 2048
    dev = torch.empty(L.lpar_host_staging_bytes_f32(N, c, eff), dtype=torch.uint8, device="cuda")
    L.lpar_allreduce_f32_host(hin, n, codec, hout, c, dev, dev.numel())
    torch.cuda.current_stream().synchronize()
    ref, used = O.allreduce_f32(xs, codec)
    assert used == codec
    for o in hout:
        assert np.array_equal(o.numpy().view(np.uint32), ref[0].view(np.uint32)), (codec, N)


def test_f32_host_threshold_on_the_whole_message(L):
    from tests.test_gpu_f32 import adversarial_f32
    n = 2048 * 6
    xs = [adversarial_f32(n, 3900 + r) for r in range(2)]
    hin = [torch.from_numpy(x.copy()).pin_memory() for x in xs]
    hout = [torch.zeros(n, dtype=torch.float32).pin_memory() for _ in range(2)]
    thr = 4 * n                                       # the whole binary32 message qualifies, a chunk would not
    dev = torch.empty(L.lpar_host_staging_bytes_f32(2, 2048 * 2, "fp8"), dtype=torch.uint8, device="cuda")
    L.lpar_allreduce_f32_host(hin, n, "fp8", hout, 2048 * 2, dev, dev.numel(), min_quant_bytes=thr)
    torch.cuda.current_stream().synchronize()
    ref, used = O.allreduce_f32(xs, "fp8", thr)
    assert used == "fp8"
    assert np.array_equal(hout[0].numpy().view(np.uint32), ref[0].view(np.uint32))


def test_f32_helper(L):
    from tests.test_gpu_f32 import adversarial_f32
    n = 2048 * 12
    xs = [adversarial_f32(n, 3950 + r) for r in range(3)]
    outs = L.allreduce_f32_host([torch.from_numpy(x.copy()).pin_memory() for x in xs], "int4", chunk=2048 * 4)
    torch.cuda.current_stream().synchronize()
    ref, _ = O.allreduce_f32(xs, "int4")
    for o in outs:
        assert o.is_pinned()
        assert np.array_equal(o.numpy().view(np.uint32), ref[0].view(np.uint32))

