"""Pins of the oracle's standalone collectives and one-shot all-reduce (CPU only).

"RCCLX: Innovating GPU communications on AMD platforms", Low-Precision
Collectives (the quantised wire serves the collectives, compute stays in FP32)
and Direct Data Access (the flat, one-shot all-reduce next to the tree).  The
pins use torch's BF16 arithmetic, inputs on each codec's grid (where quantising
is exact, so a collective reduces to a closed-form permutation or sum), the
N = 1 special case, closed-form bounds and the shard partition.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O

QCODECS = ("int4", "int3", "fp8", "mxfp4")
ALL = QCODECS + ("bf16",)


def bits(t):
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def vals(b):
    return O.bf16_bits_to_f32(b)


def randn(n, seed, scale=1.0):
    return bits(torch.randn(n, generator=torch.Generator().manual_seed(seed)) * scale)


def on_grid(codec, n, seed, spread=8):
    """BF16 values that the codec represents exactly (each block reaches its top
    code, so the stage-1 scale reproduces the grid); block scales 2^e with
    |e| <= spread (a small spread keeps sums over ranks exact in binary32)."""
    rng = np.random.default_rng(seed)
    x = np.zeros((n // 32, 32), np.float64)
    for b in range(n // 32):
        if codec in ("int4", "int3"):
            qmax = 7 if codec == "int4" else 3
            s = rng.choice([1.0, 1.25, 1.5, 1.75]) * 2.0 ** rng.integers(-spread, spread)
            k = rng.integers(-qmax, qmax + 1, 32)
            k[rng.integers(32)] = qmax * rng.choice([-1, 1])
            x[b] = k * s
        elif codec == "fp8":
            grid = [0, 0.5, 1, 1.125, 1.5, 2, 3, 7, 10, 24, 104, 240, 416, 448]     # E4M3 values
            k = rng.integers(-spread, spread)
            x[b] = rng.choice(grid, 32) * rng.choice([-1, 1], 32) * 2.0 ** k
            x[b, rng.integers(32)] = 448 * 2.0 ** k                                 # s = 2^k exactly
        elif codec == "mxfp4":
            E = rng.integers(-spread, spread)
            x[b] = rng.choice([0, 0.5, 1, 1.5, 2, 3, 4, 6], 32) * rng.choice([-1, 1], 32) * 2.0 ** E
            x[b, rng.integers(32)] = rng.choice([4.0, 6.0]) * 2.0 ** E
        else:
            x[b] = torch.from_numpy(rng.standard_normal(32)).to(torch.bfloat16).double().numpy()
    out = bits(torch.from_numpy(x.reshape(-1)).float())
    assert np.array_equal(vals(out).astype(np.float64), x.reshape(-1).astype(np.float32)), codec
    return out


def test_on_grid_inputs_round_trip_exactly():
    # the premise of the closed forms below (pinned separately by P4 and M6)
    for codec in QCODECS:
        x = on_grid(codec, 2048 * 2, 1)
        assert np.array_equal(O.decode(O.quantize(x, codec), x.size, codec), x), codec


# ---- all-gather and all-to-all: exact permutations on grid inputs --------------------------
@pytest.mark.parametrize("codec", ALL)
@pytest.mark.parametrize("N", [1, 2, 3, 5])
def test_all_gather_is_concatenation_on_grid(codec, N):
    m = 2048 * 2
    xs = [on_grid(codec, m, 10 + r) for r in range(N)]
    outs, used = O.all_gather(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(o, np.concatenate(xs))


@pytest.mark.parametrize("codec", ALL)
@pytest.mark.parametrize("N", [1, 2, 3, 4])
def test_all_to_all_is_transposition_on_grid(codec, N):
    m = 2048
    xs = [on_grid(codec, N * m, 20 + r) for r in range(N)]
    outs, _ = O.all_to_all(xs, codec)
    for j in range(N):
        assert np.array_equal(outs[j], np.concatenate([xs[r][j * m:(j + 1) * m] for r in range(N)]))


@pytest.mark.parametrize("codec", QCODECS)
def test_all_gather_and_all_to_all_off_grid_are_round_trips(codec):
    # each received segment is the decode of the sender's own wire, untouched by
    # the other ranks: exactly the single round trip of that segment
    N, m = 3, 2048 * 2
    xs = [randn(N * m, 30 + r, 10.0 ** (r - 1)) for r in range(N)]
    trips = [O.decode(O.quantize(x, codec), x.size, codec) for x in xs]
    outs, _ = O.all_to_all(xs, codec)
    for j in range(N):
        assert np.array_equal(outs[j], np.concatenate([trips[r][j * m:(j + 1) * m] for r in range(N)]))
    outs, _ = O.all_gather([x[:m] for x in xs], codec)
    for o in outs:
        assert np.array_equal(o, np.concatenate([O.decode(O.quantize(x[:m], codec), m, codec) for x in xs]))


# ---- reduce-scatter and the one-shot all-reduce --------------------------------------------
def test_bf16_reduce_scatter_matches_torch():
    N, n = 2, 2048 * 7
    a, b = randn(n, 40), randn(n, 41, 3.0)
    ref = (torch.from_numpy(vals(a)) + torch.from_numpy(vals(b))).to(torch.bfloat16)
    ref = ref.view(torch.int16).numpy().view(np.uint16)
    outs, used = O.reduce_scatter([a, b], "bf16")
    assert used == "bf16"
    for (t0, t1), o in zip(O.shard_tiles(N, n // 2048), outs):
        assert np.array_equal(o, ref[t0 * 2048:t1 * 2048])
    one, _ = O.allreduce_oneshot([a, b], "bf16")
    assert all(np.array_equal(o, ref) for o in one)


@pytest.mark.parametrize("codec", QCODECS)
@pytest.mark.parametrize("N", [2, 3, 5])
def test_reduce_scatter_on_grid_is_the_rounded_exact_sum(codec, N):
    # on-grid inputs dequantise exactly; their sums are small multiples of the
    # scales, exact in binary32 in any order, so the result is bf16(exact sum)
    n = 2048 * 5
    xs = [on_grid(codec, n, 50 + r, spread=2) for r in range(N)]
    exact = sum(vals(x).astype(np.float64) for x in xs)
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)
    ref = bits(torch.from_numpy(exact.astype(np.float32)))
    outs, _ = O.reduce_scatter(xs, codec)
    for (t0, t1), o in zip(O.shard_tiles(N, n // 2048), outs):
        assert o.size == (t1 - t0) * 2048
        assert np.array_equal(o, ref[t0 * 2048:t1 * 2048])
    one, _ = O.allreduce_oneshot(xs, codec)
    for o in one:
        assert np.array_equal(o, ref)


def test_reductions_sum_in_ascending_rank_order():
    # 2^24 + 1 rounds back to 2^24 in binary32: rank order gives 0, pairing the
    # large terms first gives 1
    big, one, nbig = O.f32_to_bf16(2.0 ** 24), O.f32_to_bf16(1.0), O.f32_to_bf16(-(2.0 ** 24))
    for order, expect in (((big, one, nbig), 0), ((big, nbig, one), one)):
        ins = [np.full(2048 * 3, v, np.uint16) for v in order]
        rs, _ = O.reduce_scatter(ins, "bf16")
        assert all(np.all(o == expect) for o in rs)
        one_shot, _ = O.allreduce_oneshot(ins, "bf16")
        assert all(np.all(o == expect) for o in one_shot)


@pytest.mark.parametrize("N", [3, 5])
def test_bf16_reductions_match_torch_fp32_sum_in_rank_order(N):
    g = torch.Generator().manual_seed(45 + N)
    n = 2048 * 4
    xs = [(torch.randn(n, generator=g) * 10.0 ** (r - 2)).to(torch.bfloat16) for r in range(N)]
    acc = torch.zeros(n, dtype=torch.float32)
    for x in xs:
        acc = acc + x.float()
    ref = bits(acc)
    ins = [x.view(torch.int16).numpy().view(np.uint16) for x in xs]
    rs, _ = O.reduce_scatter(ins, "bf16")
    for (t0, t1), o in zip(O.shard_tiles(N, n // 2048), rs):
        assert np.array_equal(o, ref[t0 * 2048:t1 * 2048])
    one_shot, _ = O.allreduce_oneshot(ins, "bf16")
    assert all(np.array_equal(o, ref) for o in one_shot)


def test_shard_partition_is_the_floor_split():
    assert O.shard_tiles(3, 10) == [(0, 3), (3, 6), (6, 10)]
    assert O.shard_tiles(8, 5) == [(0, 0), (0, 1), (1, 1), (1, 2), (2, 3), (3, 3), (3, 4), (4, 5)]


@pytest.mark.parametrize("codec", QCODECS)
def test_n1_reductions_are_one_round_trip(codec):
    x = randn(2048 * 3, 60)
    trip = O.decode(O.quantize(x, codec), x.size, codec)
    trip = np.where(trip == 0x8000, 0, trip)            # +0 + (-0) = +0 in the FP32 sum
    for fn in (O.reduce_scatter, O.allreduce_oneshot):
        outs, _ = fn([x], codec)
        assert np.array_equal(outs[0], trip)


@pytest.mark.parametrize("codec", QCODECS)
def test_oneshot_error_bound_has_one_quantisation_stage(codec):
    # |out - exact| <= sum_r (stage-1 error of rank r) + FP32 sum error + BF16
    # half-ulp; no second-stage term, unlike the two-shot all-reduce
    N, n = 4, 2048 * 2
    xs = [randn(n, 70 + r, 2.0 ** r) for r in range(N)]
    one, _ = O.allreduce_oneshot(xs, codec)
    out = vals(one[0]).astype(np.float64)
    x64 = [vals(x).astype(np.float64) for x in xs]
    tb = O.tile_bytes(codec)
    v64 = []
    for x in xs:                                                    # stage-1 values in binary32
        w = O.quantize(x, codec)
        v64.append(np.concatenate([O.dequant_tile(w[t * tb:(t + 1) * tb], codec) for t in range(n // 2048)])
                   .astype(np.float64))
    stage1 = sum(np.abs(a - b) for a, b in zip(x64, v64))
    fp32 = (N - 1) * 2.0 ** -24 * sum(np.abs(t) for t in v64)
    bound = stage1 + fp32 + 2.0 ** -8 * np.abs(out)
    assert np.all(np.abs(out - sum(x64)) <= bound)


def test_thresholds():
    thr = 1 << 20
    N = 2
    n_small = thr // 2 - 2048                       # 2n just below 1 MiB
    xs = [randn(n_small, 80 + r) for r in range(N)]
    assert O.reduce_scatter(xs, "int3", thr)[1] == "bf16"
    assert O.allreduce_oneshot(xs, "int3", thr)[1] == "bf16"
    assert O.all_gather(xs, "int3", thr)[1] == "bf16"
    # all-to-all measures the whole per-rank message (N segments)
    m = thr // 4                                    # 2 * N * m = 1 MiB
    ys = [randn(N * m, 90 + r) for r in range(N)]
    assert O.all_to_all(ys, "int3", thr)[1] == "int3"
    assert O.all_gather([y[:m] for y in ys], "int3", thr)[1] == "bf16"
