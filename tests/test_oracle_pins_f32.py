"""Pins of the oracle's all-reduce of FP32 messages (CPU only).

"RCCLX: Innovating GPU communications on AMD platforms", Low-Precision
Collectives: FP32 or BF16 inputs, FP8 on the wire for up to 4:1 against FP32,
computation in FP32.  The result of an FP32 message is the dequantised gathered
value itself (binary32).  Pins: the printed ratio, numpy's binary32 sums in
rank order, exact-rational brute force of the codes of 24-bit inputs, on-grid
round trips, a closed-form bound and the threshold.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O
from tests import brute as B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
QCODECS = ("int4", "int3", "fp8", "mxfp4")
TWO = Fraction(2)


def f32s(n, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(n) * scale).astype(np.float32)


def test_fp8_is_four_to_one_against_fp32():
    F = json.load(open(os.path.join(GOLDEN, "page_facts.json")))
    code_bytes = 2048 / 2048                         # one E4M3 byte per element
    assert 4 / code_bytes == F["fp8_compression_vs_fp32"]["value"] == 4
    # with the per-32 binary32 scales the FP8 wire is 8192 / 2304 = 3.56 : 1 against FP32
    assert round(2048 * 4 / O.tile_bytes("fp8"), 2) == 3.56


@pytest.mark.parametrize("N", [2, 3, 5])
def test_passthrough_is_numpy_float32_sum_in_rank_order(N):
    n = 2048 * 2
    xs = [f32s(n, 10 + r, 10.0 ** (r - 2)) for r in range(N)]
    acc = np.zeros(n, np.float32)
    for x in xs:
        acc = (acc + x).astype(np.float32)
    outs, used = O.allreduce_f32(xs, "bf16")
    assert used == "bf16"
    for o in outs:
        assert np.array_equal(o, acc)


def test_passthrough_rank_order_trap():
    big, one = np.float32(2.0 ** 24), np.float32(1.0)
    for order, expect in (((big, one, -big), 0.0), ((big, -big, one), 1.0)):
        ins = [np.full(2048, v, np.float32) for v in order]
        outs, _ = O.allreduce_f32(ins, "bf16")
        assert np.all(outs[0] == expect)


@pytest.mark.parametrize("codec", ["int4", "int3"])
def test_int_codes_of_24_bit_inputs_match_exact_rationals(codec):
    bits = 4 if codec == "int4" else 3
    rng = np.random.default_rng(20 + bits)
    for trial in range(400):
        wide = trial % 4 != 0                        # saturating and subnormal scales included
        x = (rng.standard_normal(32) * 2.0 ** rng.integers(-30, 30) if wide else
             rng.standard_normal(32) * 2.0 ** rng.integers(-10, 10)).astype(np.float32)
        if not wide:                                 # exact ties of the grid with full 24-bit values
            s = np.float32(O.f16_to_f32(O.f32_to_f16(np.max(np.abs(x)) / (2 ** (bits - 1) - 1))))
            x[1:8] = (np.array([0.5, 1.5, -2.5, 0.5, -0.5, 1.5, -1.5], np.float32) * s).astype(np.float32)
        sb, codes = O.quant_block_int(x, bits)
        s_ref, c_ref = B.quant_block_int([Fraction(float(v)) for v in x], bits)
        assert Fraction(O.f16_to_f32(sb)) == s_ref
        assert list(codes) == c_ref


def test_fp8_and_mxfp4_codes_of_24_bit_inputs_match_exact_rationals():
    rng = np.random.default_rng(30)
    for _ in range(300):
        x = (rng.standard_t(3, 32) * 2.0 ** rng.integers(-40, 40)).astype(np.float32)
        s, codes = O.quant_block_fp8(x)
        s_ref, c_ref = B.quant_block_fp8([Fraction(float(v)) for v in x])
        assert Fraction(s) == s_ref and list(codes) == c_ref
        sc, codes = O.quant_block_mxfp4(x)
        E, c_ref = B.quant_block_mxfp4([Fraction(float(v)) for v in x], [bool(np.signbit(v)) for v in x])
        assert sc == E + 127 and list(codes) == c_ref


def on_grid_f32(codec, n, seed):
    rng = np.random.default_rng(seed)
    x = np.zeros((n // 32, 32), np.float64)
    for b in range(n // 32):
        if codec in ("int4", "int3"):
            qmax = 7 if codec == "int4" else 3
            s = O.f16_to_f32(O.f32_to_f16(rng.uniform(0.5, 2) * 2.0 ** rng.integers(-12, 12)))
            k = rng.integers(-qmax, qmax + 1, 32)
            k[rng.integers(32)] = qmax
            x[b] = k * s
        elif codec == "fp8":
            e = rng.integers(-20, 20)
            x[b] = rng.choice([0, 0.25, 1, 1.125, 3, 13, 104, 240, 448], 32) * 2.0 ** e
            x[b, 0] = 448 * 2.0 ** e
        else:
            E = rng.integers(-30, 30)
            x[b] = rng.choice([0, 0.5, 1, 1.5, 2, 3, 4, 6], 32) * rng.choice([-1, 1], 32) * 2.0 ** E
            x[b, 0] = 6 * 2.0 ** E
    out = x.reshape(-1).astype(np.float32)
    assert np.array_equal(out.astype(np.float64), x.reshape(-1))
    return out


@pytest.mark.parametrize("codec", QCODECS)
def test_on_grid_fp32_messages_round_trip_exactly(codec):
    x = on_grid_f32(codec, 2048 * 3, 40)
    outs, used = O.allreduce_f32([x], codec)
    assert used == codec
    assert np.array_equal(outs[0], x)


@pytest.mark.parametrize("codec", QCODECS)
def test_end_to_end_error_bound(codec):
    N, n = 4, 2048 * 2
    xs = [f32s(n, 50 + r, 3.0 ** r) for r in range(N)]
    outs, _ = O.allreduce_f32(xs, codec)
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    tb = O.tile_bytes(codec)
    wires = [np.concatenate([O.quant_tile(x[t * 2048:(t + 1) * 2048], codec) for t in range(n // 2048)]) for x in xs]
    v = [np.concatenate([O.dequant_tile(w[t * tb:(t + 1) * tb], codec) for t in range(n // 2048)]).astype(np.float64)
         for w in wires]
    x64 = [x.astype(np.float64) for x in xs]
    stage1 = sum(np.abs(a - b) for a, b in zip(x64, v))             # realised stage-1 errors
    fp32 = (N - 1) * 2.0 ** -24 * sum(np.abs(t) for t in v)
    acc = sum(v)                                                    # within fp32 of the binary32 sum
    amax = np.max(np.abs(acc.reshape(-1, 32)), axis=1).repeat(32)
    # one more quantisation stage of the sums: half a grid step of the block (INT:
    # s/2 = amax/(2 qmax) up to binary16 rounding; FP8: 2^-4 relative plus the
    # subnormal grid; MXFP4: the saturation distance of at most 2^(E+1) <= amax/2)
    stage2 = {"int4": amax / 14 * 1.001, "int3": amax / 6 * 1.001, "fp8": np.abs(acc) * 2.0 ** -4 + amax * 2.0 ** -18,
              "mxfp4": amax / 2}[codec]
    out = outs[0].astype(np.float64)
    assert np.all(np.abs(out - sum(x64)) <= stage1 + fp32 + stage2 + fp32)


def test_threshold_counts_fp32_bytes():
    thr = 1 << 20
    n = thr // 4                                     # 4n = 1 MiB: quantised
    xs = [f32s(n, 60 + r) for r in range(2)]
    assert O.allreduce_f32(xs, "fp8", thr)[1] == "fp8"
    ys = [x[:n - 2048] for x in xs]
    assert O.allreduce_f32(ys, "fp8", thr)[1] == "bf16"
