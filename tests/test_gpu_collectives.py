"""CUDA collectives (reduce-scatter, all-gather, all-to-all, one-shot all-reduce)
against the CPU oracle, bit for bit (needs a B200).

Inputs are seeded: adversarial BF16 blocks (the same generator as the all-reduce
parity tests) for odd ranks, Gaussian values at rank-dependent scales for even
ranks.  Every device buffer the library writes has guard bands, checked after
each call; expected values come only from the oracle.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as O
from tests.test_gpu_parity import Guarded, adversarial_bf16, host_u16, random_bf16, to_device

pytestmark = pytest.mark.gpu

CODECS = ("int4", "int3", "fp8", "mxfp4", "bf16")


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


def inputs(N, n, seed):
    return [adversarial_bf16(n, seed + r) if r % 2 else random_bf16(n, seed + 100 + r, 10.0 ** (r - 2))
            for r in range(N)]


def run(L, op, xs, size, codec, out_sizes, min_quant_bytes=0):
    N = len(xs)
    ins = [to_device(x) for x in xs]
    outs = [Guarded(2 * k, fill=0x00) for k in out_sizes]
    n_msg = N * size if op == "all_to_all" else size
    eff = L.lpar_effective_codec(n_msg, codec, min_quant_bytes)
    need = L.lpar_collective_workspace_bytes(op, N, size, eff)
    ws = Guarded(need)
    fn = getattr(L, "lpar_" + op)
    fn([g.ptr() for g in ins], size, codec, [g.ptr() for g in outs], ws.ptr() if need else 0, ws.nbytes,
       min_quant_bytes=min_quant_bytes)
    torch.cuda.synchronize()
    for g in ins + outs + [ws]:
        g.check()
    return [host_u16(g) for g in outs], eff


# Seeded random cases: operation, codec, N in 1..8, 1..24 tiles, a threshold
# either side of the message; adversarial and random inputs.
@pytest.mark.parametrize("case", range(36))
def test_collectives_random_cases(L, case):
    rng = np.random.default_rng(9500 + case)
    op = ("reduce_scatter", "all_gather", "all_to_all")[rng.integers(3)]
    codec = CODECS[rng.integers(len(CODECS))]
    N = int(rng.integers(1, 9))
    tiles = int(rng.integers(1, 25))
    size = tiles * 2048
    n_msg = N * size if op == "all_to_all" else size
    thr = (0, 2 * n_msg, 2 * n_msg + 2)[rng.integers(3)]
    xs = inputs(N, n_msg, int(rng.integers(1 << 20)))
    if op == "reduce_scatter":
        sizes = [(t1 - t0) * 2048 for t0, t1 in O.shard_tiles(N, tiles)]
        ref, used = O.reduce_scatter(xs, codec, thr)
    elif op == "all_gather":
        sizes = [N * size] * N
        ref, used = O.all_gather(xs, codec, thr)
    else:
        sizes = [N * size] * N
        ref, used = O.all_to_all(xs, codec, thr)
    outs, eff = run(L, op, xs, size, codec, sizes, thr)
    assert eff == used
    for j, (o, r) in enumerate(zip(outs, ref)):
        assert np.array_equal(o, r), (op, codec, N, tiles, thr, j)


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles", [(1, 5), (2, 9), (3, 13), (5, 3), (8, 21)])
def test_reduce_scatter_matches_oracle(L, codec, N, tiles):
    n = tiles * 2048
    xs = inputs(N, n, 1000 + 10 * N)
    sizes = [(t1 - t0) * 2048 for t0, t1 in O.shard_tiles(N, tiles)]
    outs, _ = run(L, "reduce_scatter", xs, n, codec, sizes)
    ref, used = O.reduce_scatter(xs, codec)
    assert used == codec
    for j, (o, r) in enumerate(zip(outs, ref)):
        assert np.array_equal(o, r), (codec, N, j)


# The reductions' forms around the limit of the rank-parallel tile form (256
# tiles per rank, 512 for FP8): at it the tile form, just above it the
# persistent forms with a ragged last chunk.
@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "mxfp4"])
@pytest.mark.parametrize("N", [1, 3, 8])
@pytest.mark.parametrize("extra", [0, 1, 3])
def test_reductions_around_the_tile_limit(L, codec, N, extra):
    tiles = (512 if codec == "fp8" else 256) + extra
    n = tiles * 2048
    xs = inputs(N, n, 1500 + 10 * N + extra)
    sizes = [(t1 - t0) * 2048 for t0, t1 in O.shard_tiles(N, tiles)]
    outs, _ = run(L, "reduce_scatter", xs, n, codec, sizes)
    ref, used = O.reduce_scatter(xs, codec)
    assert used == codec
    for j, (o, r) in enumerate(zip(outs, ref)):
        assert np.array_equal(o, r), (codec, N, tiles, j)
    ins = [to_device(x) for x in xs]
    outs1 = [Guarded(2 * n, fill=0x00) for _ in range(N)]
    ws = Guarded(L.lpar_workspace_bytes(N, n, codec))
    L.lpar_allreduce([g.ptr() for g in ins], n, codec, [g.ptr() for g in outs1], ws.ptr(), ws.nbytes,
                     schedule="one_shot")
    torch.cuda.synchronize()
    for g in ins + outs1 + [ws]:
        g.check()
    ref1, _ = O.allreduce_oneshot(xs, codec)
    for o in outs1:
        assert np.array_equal(host_u16(o), ref1[0]), (codec, N, tiles)


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles", [(1, 5), (2, 9), (3, 6), (5, 2), (8, 7)])
def test_all_gather_matches_oracle(L, codec, N, tiles):
    m = tiles * 2048
    xs = inputs(N, m, 2000 + 10 * N)
    outs, _ = run(L, "all_gather", xs, m, codec, [N * m] * N)
    ref, used = O.all_gather(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(o, ref[0])


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles", [(1, 5), (2, 3), (3, 2), (5, 1), (8, 3)])
def test_all_to_all_matches_oracle(L, codec, N, tiles):
    m = tiles * 2048
    xs = inputs(N, N * m, 3000 + 10 * N)
    outs, _ = run(L, "all_to_all", xs, m, codec, [N * m] * N)
    ref, used = O.all_to_all(xs, codec)
    assert used == codec
    for j, (o, r) in enumerate(zip(outs, ref)):
        assert np.array_equal(o, r), (codec, N, j)


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N", [1, 2, 3, 8])
def test_one_shot_allreduce_matches_oracle(L, codec, N):
    tiles = 9
    n = tiles * 2048
    xs = inputs(N, n, 4000 + N)
    ins = [to_device(x) for x in xs]
    outs = [Guarded(2 * n, fill=0x00) for _ in range(N)]
    ws = Guarded(L.lpar_workspace_bytes(N, n, codec))
    L.lpar_allreduce([g.ptr() for g in ins], n, codec, [g.ptr() for g in outs], ws.ptr(), ws.nbytes,
                     schedule="one_shot")
    torch.cuda.synchronize()
    for g in ins + outs + [ws]:
        g.check()
    ref, used = O.allreduce_oneshot(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(host_u16(o), ref[0])


def test_thresholds_send_small_messages_to_bf16(L):
    thr = 1 << 20
    N, n = 2, (1 << 20) // 2 - 2048
    xs = inputs(N, n, 5000)
    outs, eff = run(L, "reduce_scatter", xs, n, "int3", [(t1 - t0) * 2048 for t0, t1 in O.shard_tiles(N, n // 2048)],
                    min_quant_bytes=thr)
    ref, used = O.reduce_scatter(xs, "int3", thr)
    assert eff == used == "bf16"
    assert all(np.array_equal(o, r) for o, r in zip(outs, ref))
    m = (1 << 20) // 4                                   # all-to-all: 2 * N * m = 1 MiB, quantised
    ys = inputs(N, N * m, 5100)
    outs, eff = run(L, "all_to_all", ys, m, "int3", [N * m] * N, min_quant_bytes=thr)
    ref, used = O.all_to_all(ys, "int3", thr)
    assert eff == used == "int3"
    assert all(np.array_equal(o, r) for o, r in zip(outs, ref))


def test_python_helpers_match_oracle(L):
    N, n = 3, 2048 * 6
    xs = inputs(N, n, 6000)
    dxs = [torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in xs]
    rs = L.reduce_scatter(dxs, "int4")
    ref, _ = O.reduce_scatter(xs, "int4")
    assert all(np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), r) for o, r in zip(rs, ref))
    ag = L.all_gather(dxs, "fp8")
    ref, _ = O.all_gather(xs, "fp8")
    assert all(np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), ref[0]) for o in ag)
    a2a = L.all_to_all(dxs, "mxfp4")
    ref, _ = O.all_to_all(xs, "mxfp4")
    assert all(np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), r) for o, r in zip(a2a, ref))


# ---------------------------------------------------------------------------
# Full size, in the launch configuration the bench times: 256 MiB per rank,
# checked on 256 seeded random tiles plus the first and the last (tiles are
# independent; for all-to-all and all-gather a received tile depends only on
# the sender's tile).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("op", ["reduce_scatter", "one_shot", "all_gather", "all_to_all"])
def test_large_sampled_tiles(L, op):
    N, n = 4, 128 * 1024 * 1024
    w = W.Workload("large_collective", N=N, n=n, dist="normal", sigma=0.02, seed=7, codecs=("int4",))
    xs = W.make_inputs(w, "cuda")
    T = n // 2048
    rng = np.random.default_rng(8)
    tiles = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 256, replace=False)]))
    for codec in ("int3", "mxfp4"):
        if op in ("reduce_scatter", "one_shot"):
            outs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(N)]
            ws = torch.empty(L.lpar_workspace_bytes(N, n, codec), dtype=torch.uint8, device="cuda")
            if op == "one_shot":
                L.lpar_allreduce(xs, n, codec, outs, ws, ws.numel(), schedule="one_shot")
            else:
                L.lpar_reduce_scatter(xs, n, codec, outs, ws, ws.numel())
            torch.cuda.synchronize()
            idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
            sample = [x[idx].view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
            ref, _ = O.allreduce_oneshot(sample, codec)
            shards = O.shard_tiles(N, T)
            for k, t in enumerate(tiles):
                if op == "one_shot":
                    for o in outs:
                        got = o[t * 2048:(t + 1) * 2048].view(torch.int16).cpu().numpy().view(np.uint16)
                        assert np.array_equal(got, ref[0][k * 2048:(k + 1) * 2048]), (op, codec, t)
                else:
                    j = next(j for j, (t0, t1) in enumerate(shards) if t0 <= t < t1)
                    loc = t - shards[j][0]
                    got = outs[j][loc * 2048:(loc + 1) * 2048].view(torch.int16).cpu().numpy().view(np.uint16)
                    assert np.array_equal(got, ref[0][k * 2048:(k + 1) * 2048]), (op, codec, t)
        else:
            m = n // N                                        # all-to-all: N segments of m; all-gather: m each
            src = xs if op == "all_to_all" else [x[:m] for x in xs]
            outs = [torch.empty(N * m, dtype=torch.bfloat16, device="cuda") for _ in range(N)]
            ws = torch.empty(L.lpar_collective_workspace_bytes(op, N, m, codec), dtype=torch.uint8, device="cuda")
            getattr(L, "lpar_" + op)(src, m, codec, outs, ws, ws.numel())
            torch.cuda.synchronize()
            mt = m // 2048
            stiles = np.unique(np.concatenate([[0, (len(src[0]) // 2048) - 1],
                                               rng.choice(len(src[0]) // 2048, 128, replace=False)]))
            for r in range(N):
                idx = torch.from_numpy((stiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
                sample = src[r][idx].view(torch.int16).cpu().numpy().view(np.uint16)
                trip = O.decode(O.quantize(sample, codec), sample.size, codec)
                for k, t in enumerate(stiles):
                    if op == "all_to_all":
                        j, tl = t // mt, t % mt
                        dsts = [(j, r * mt + tl)]
                    else:
                        dsts = [(j, r * mt + t) for j in range(N)]
                    for j, dt in dsts:
                        got = outs[j][dt * 2048:(dt + 1) * 2048].view(torch.int16).cpu().numpy().view(np.uint16)
                        assert np.array_equal(got, trip[k * 2048:(k + 1) * 2048]), (op, codec, r, t)
        del outs, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N", [3, 5])
def test_all_gather_reduced_grid_ragged(L, N):
    """The all-gather from 64 MiB of input runs on fewer CTAs (2 per SM for
    N <= 3, 1 for N = 4..7); here with a ragged last chunk (tiles % 4 == 3),
    sampled tiles against the oracle's round trip at every destination."""
    mt = -(-(64 << 20) // (N * 4096))
    mt += (3 - mt % 4) % 4
    m = mt * 2048
    assert N * m * 2 >= (64 << 20) and mt % 4 == 3
    w = W.Workload("capped_all_gather", N=N, n=m, dist="student_t", nu=3, seed=11, codecs=("int4",))
    xs = W.make_inputs(w, "cuda")
    rng = np.random.default_rng(12)
    stiles = np.unique(np.concatenate([np.arange(mt - 5, mt), rng.choice(mt, 64, replace=False)]))
    idx = torch.from_numpy((stiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
    for codec in ("int4", "fp8"):
        outs = [torch.empty(N * m, dtype=torch.bfloat16, device="cuda") for _ in range(N)]
        ws = torch.empty(L.lpar_collective_workspace_bytes("all_gather", N, m, codec), dtype=torch.uint8,
                         device="cuda")
        L.lpar_all_gather(xs, m, codec, outs, ws, ws.numel())
        torch.cuda.synchronize()
        for r in range(N):
            sample = xs[r][idx].view(torch.int16).cpu().numpy().view(np.uint16)
            trip = O.decode(O.quantize(sample, codec), sample.size, codec)
            for j in range(N):
                got = outs[j][r * m:(r + 1) * m][idx].view(torch.int16).cpu().numpy().view(np.uint16)
                assert np.array_equal(got, trip), (codec, N, r, j)
        del outs, ws
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# The cross-process all-reduce on the GPU: the library's stages with NCCL
# collectives.  Only one GPU is available, so this runs one process (the
# exchanges are NCCL calls on one rank); the orchestration at 2-4 ranks is
# covered on CPU with gloo (tests/test_distributed_host.py).
# ---------------------------------------------------------------------------
def test_cross_process_allreduce_one_rank_nccl(L):
    import socket
    import torch.distributed as dist
    from quantized_precision_all_b200.distributed import DistributedAllreduce
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        ar = DistributedAllreduce()
        for codec in ("int3", "int4", "fp8", "mxfp4", "bf16"):
            x = adversarial_bf16(2048 * 6, 4200)
            out = ar.allreduce(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16), codec)
            torch.cuda.synchronize()
            ref, _ = O.allreduce([x], codec)
            assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ref[0]), codec
    finally:
        dist.destroy_process_group()
