"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each test names the pin it checks.  None of them re-types the oracle's own
formula: they use the printed page facts, hand-derived worked examples, exact
rational brute force (tests/brute.py), library conversions (numpy, torch),
closed-form error bounds and invariants.
"""
import json
import os
import random
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import brute as B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def facts():
    with open(os.path.join(GOLDEN, "page_facts.json")) as f:
        return json.load(f)


def f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


def bf16_values_in(lo, hi):
    """Every BF16 bit pattern whose value lies in [lo, hi]."""
    out = []
    for bits in range(0x10000):
        if (bits & 0x7F80) == 0x7F80:
            continue
        v = B.bf16_exact(bits)
        if lo <= v <= hi:
            out.append(bits)
    return out


# ---- P1-P3: the printed sizes and ratios -------------------------------------
def test_p1_tile_bytes_match_pages():
    F = facts()
    assert O.tile_bytes("int4") == F["int4_tile_bytes"]["value"] == 1152
    assert O.tile_bytes("int3") == F["int3_tile_bytes"]["value"] == 896
    # 2048 elements per tile: codes plus 64 binary16 scales
    assert O.tile_bytes("int4") == 2048 * 4 // 8 + 64 * 2
    assert O.tile_bytes("int3") == 2048 * 3 // 8 + 64 * 2
    assert O.wire_bytes("int3", 2048 * 5) == 5 * 896


def test_p2_int3_saving_is_22_percent():
    F = facts()
    saving = 1 - O.tile_bytes("int3") / O.tile_bytes("int4")
    assert round(100 * saving) == F["int3_vs_int4_reduction_percent"]["value"]


def test_p3_fp8_ratio_and_wire_ratios():
    F = facts()
    code_bytes_per_elem = (O.tile_bytes("fp8") - 64 * 4) / 2048
    assert 4 / code_bytes_per_elem == F["fp8_compression_vs_fp32"]["value"]
    # with one binary32 scale per 32 elements: 3.56:1 vs FP32, 1.78:1 vs BF16
    assert abs(2048 * 4 / O.tile_bytes("fp8") - 128 / 36) < 1e-12
    assert abs(2048 * 2 / O.tile_bytes("fp8") - 64 / 36) < 1e-12
    assert O.e4m3_to_f32(0x7E) == F["e4m3_max_finite"]["value"]


# ---- hand-derived worked examples -------------------------------------------
def test_worked_int4_block_unit_scale():
    # absmax 7 -> 7/7 = 1 -> s = 1.0 (binary16 0x3C00); q = RNE(x): ties go even
    x = [7, -3.5, 1.75, 0.5, 1.5, 2.5, -2.5, 6.5, -7] + [0] * 23
    sb, codes = O.quant_block_int(np.array(x, np.float32), 4)
    assert sb == 0x3C00
    assert list(codes[:9]) == [15, 4, 10, 8, 10, 10, 6, 14, 1]
    assert all(c == 8 for c in codes[9:])


def test_worked_int4_block_rounded_scale():
    # absmax 1 -> fl32(1/7) -> binary16: 2^-3 * (1 + 146/1024) = 1170/8192, bits 0x3092
    s = Fraction(1170, 8192)
    x = [1.0, 0.5, -0.5, 0.25, float(Fraction(4095, 8192)), float(Fraction(2925, 8192)),
         float(-Fraction(1755, 8192))] + [0.0] * 25
    sb, codes = O.quant_block_int(np.array(x, np.float32), 4)
    assert sb == 0x3092 and Fraction(O.f16_to_f32(sb)) == s
    # 1/s = 7.0017 -> 7; 0.5/s = 3.5009 -> 4 (not a tie); 0.25/s = 1.75 -> 2;
    # 4095/8192 = 3.5 s exactly -> tie -> 4; 2925/8192 = 2.5 s -> 2; -1755/8192 = -1.5 s -> -2
    assert list(codes[:7]) == [15, 12, 4, 10, 12, 10, 6]


def test_worked_int3_tile_packing():
    # block 0: absmax 3 -> s = 1; q = 3, -2, 2, 0, -3, 1 -> codes 7, 2, 6, 4, 1, 5, then 4s
    x = np.zeros(2048, np.float32)
    x[:6] = [3, -1.5, 2.5, 0.5, -3, 1]
    tile = O.quant_tile(x, "int3")
    assert tile.size == 896
    assert tile[0] == 0x2B          # (3) | (2<<2) | (2<<4) | (0<<6)
    assert tile[1] == 0x05          # (1) | (1<<2) | (0<<4) | (0<<6)
    assert all(tile[2:512] == 0)    # code 4 has low bits 00 ...
    assert tile[512] == 0xED        # high bits of codes 7,2,6,4,1,5,4,4 = 1,0,1,1,0,1,1,1
    assert all(tile[513:768] == 0xFF)   # ... and high bit 1
    assert tile[768] == 0x00 and tile[769] == 0x3C      # scale of block 0, little-endian
    assert all(tile[770:] == 0)     # all-zero blocks have scale 0


def test_worked_fp8_block():
    # absmax 448 -> s = 1, 1/s = 1: the codes are E4M3 of the inputs themselves
    x = [448, 1.0, 17.0, -2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, -300] + [0] * 25
    s, codes = O.quant_block_fp8(np.array(x, np.float32))
    assert s == 1.0
    # 17 is a tie of 16 and 18 -> 16 (even mantissa); 2^-10 ties 0 and 2^-9 -> 0;
    # 300 lies between 288 and 320 -> 288
    assert list(codes[:7]) == [0x7E, 0x38, 0x58, 0x81, 0x00, 0x01, 0xF9]


def test_worked_allreduce_two_ranks():
    # rank 0 block 0 = [7, 1, 2], rank 1 = [-7, 3, 0]; both have s = 1, so the FP32
    # sums are [0, 4, 2].  Requantised: absmax 4 -> s2 = 1170/2048; 4/s2 = 7.0017 -> 7,
    # 2/s2 = 3.5009 -> 4.  Decoded: 7 s2 = 3.99902 -> BF16 4.0 (0x4080);
    # 4 s2 = 2.28516 -> BF16 2.28125 (0x4012).
    a = np.zeros(2048, np.float32); a[:3] = [7, 1, 2]
    b = np.zeros(2048, np.float32); b[:3] = [-7, 3, 0]
    ins = [np.array([O.f32_to_bf16(v) for v in a], np.uint16),
           np.array([O.f32_to_bf16(v) for v in b], np.uint16)]
    outs, used = O.allreduce(ins, "int4")
    assert used == "int4"
    for o in outs:
        assert list(o[:3]) == [0x0000, 0x4080, 0x4012]
        assert all(o[3:] == 0)


# ---- P4: on-grid round trip -------------------------------------------------
@pytest.mark.parametrize("bits", [4, 3])
def test_p4_on_grid_round_trip_int(bits):
    rng = random.Random(40 + bits)
    qmax = 2 ** (bits - 1) - 1
    for _ in range(300):
        e = rng.randint(-14, 14)
        m = rng.randint(1024, 2047)
        s = m * 2.0 ** (e - 10)                          # a normal binary16 value
        k = [rng.randint(-qmax, qmax) for _ in range(32)]
        k[rng.randrange(32)] = qmax * rng.choice([-1, 1])
        x = np.array([ki * s for ki in k], np.float32)
        sb, codes = O.quant_block_int(x, bits)
        assert O.f16_to_f32(sb) == s
        assert [int(c) - 2 ** (bits - 1) for c in codes] == k
        assert [O.dequant_int(c, bits, sb) for c in codes] == list(x)


def test_p4_on_grid_round_trip_fp8():
    rng = random.Random(44)
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    for _ in range(300):
        k = rng.randint(-60, 60)
        codes = [rng.choice(finite) for _ in range(32)]
        codes[rng.randrange(32)] = rng.choice([0x7E, 0xFE])     # absmax 448 * 2^k
        x = np.array([O.e4m3_to_f32(c) * 2.0 ** k for c in codes], np.float32)
        s, got = O.quant_block_fp8(x)
        assert s == 2.0 ** k
        # +0 and -0 both decode to zero; compare values, not the sign of zero
        assert [O.dequant_fp8(g, s) for g in got] == list(x)


# ---- P5: all-zero block -----------------------------------------------------
def test_p5_all_zero_blocks():
    z = np.zeros(32, np.float32)
    for bits in (4, 3):
        sb, codes = O.quant_block_int(z, bits)
        assert sb == 0 and all(codes == 2 ** (bits - 1))
        assert O.dequant_int(codes[0], bits, sb) == 0.0
    s, codes = O.quant_block_fp8(z)
    assert s == 0.0 and all(codes == 0)
    for codec in ("int4", "int3", "fp8", "bf16"):
        out = O.decode(O.quantize(np.zeros(4096, np.uint16), codec), 4096, codec)
        assert all(out == 0)


# ---- P6: per-stage error bound ----------------------------------------------
def _rand_block(rng, scale):
    return np.array([f32(rng.gauss(0, 1) * scale) for _ in range(32)], np.float32)


@pytest.mark.parametrize("bits", [4, 3])
def test_p6_int_error_at_most_half_scale(bits):
    rng = random.Random(60 + bits)
    for i in range(2000):
        x = _rand_block(rng, 10.0 ** rng.uniform(-3, 3))
        if i % 7 == 0:
            x[rng.randrange(32)] *= 50                   # an outlier
        sb, codes = O.quant_block_int(x, bits)
        s = Fraction(O.f16_to_f32(sb))
        assert 2 ** -14 <= s < 65504                   # stays a normal binary16 here
        for xi, c in zip(x, codes):
            v = Fraction(O.dequant_int(c, bits, sb))
            assert abs(Fraction(float(xi)) - v) <= s / 2


def test_p6_fp8_error_bound():
    rng = random.Random(66)
    for _ in range(2000):
        x = _rand_block(rng, 10.0 ** rng.uniform(-20, 20))
        s, codes = O.quant_block_fp8(x)
        for xi, c in zip(x, codes):
            v = Fraction(O.dequant_fp8(c, s))
            X = Fraction(float(xi))
            bound = abs(X) / 16 + Fraction(s) / 1024 + abs(X) * Fraction(1, 2 ** 21)
            assert abs(X - v) <= bound


# ---- P7: idempotence; N = 1 all-reduce is one round trip ---------------------
@pytest.mark.parametrize("codec", ["int4", "int3", "fp8"])
def test_p7_requantising_a_decoded_tile_is_identity(codec):
    rng = np.random.default_rng(70)
    for _ in range(20):
        x = (rng.standard_normal(2048) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        t1 = O.quant_tile(x, codec)
        t2 = O.quant_tile(O.dequant_tile(t1, codec), codec)
        if codec == "fp8":
            # decoded FP8 values re-encode to the same codes when the block's
            # absmax code is 448 (s is then recomputed exactly)
            assert np.array_equal(O.dequant_tile(t2, codec), O.dequant_tile(t1, codec))
        else:
            assert np.array_equal(t1, t2)


@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "bf16"])
def test_p7_single_rank_equals_one_round_trip(codec):
    x = torch.randn(8192, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    outs, _ = O.allreduce([bits], codec)
    one_trip = O.decode(O.quantize(bits, codec), bits.size, codec)
    assert np.array_equal(outs[0], one_trip)


# ---- P8: antisymmetry -------------------------------------------------------
@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "bf16"])
def test_p8_opposite_ranks_cancel_to_positive_zero(codec):
    x = torch.randn(4096, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    a = x.view(torch.int16).numpy().view(np.uint16)
    b = (-x).view(torch.int16).numpy().view(np.uint16)
    outs, _ = O.allreduce([a, b], codec)
    for o in outs:
        assert np.all(o == 0)        # +0.0 everywhere, never -0.0


# ---- P9: exact-rational brute force -----------------------------------------
@pytest.mark.parametrize("bits", [4, 3])
def test_p9_brute_force_int_every_bf16_in_range(bits):
    rng = random.Random(90 + bits)
    base = [B.bf16_exact(O.f32_to_bf16(rng.uniform(-3, 3))) for _ in range(32)]
    base[5] = Fraction(3)                                # absmax 3 unless x0 wins
    vals = bf16_values_in(-8, 8)
    for bits0 in vals:
        xs = list(base)
        xs[0] = B.bf16_exact(bits0)
        s_ref, codes_ref = B.quant_block_int(xs, bits)
        sb, codes = O.quant_block_int(np.array([float(v) for v in xs], np.float32), bits)
        assert Fraction(O.f16_to_f32(sb)) == s_ref
        assert list(codes) == codes_ref, (hex(bits0), float(xs[0]))


@pytest.mark.parametrize("bits", [4, 3])
def test_p9_brute_force_int_fp32_sums_and_ties(bits):
    """Stage-2 inputs are arbitrary binary32 sums; include exact and near ties."""
    rng = random.Random(95 + bits)
    for i in range(3000):
        xs = [B.rn32(Fraction(rng.gauss(0, 1)) * Fraction(2) ** rng.randint(-20, 20)) for _ in range(32)]
        if i % 3 == 0:
            # plant exact ties (k + 1/2) * s and neighbours one ulp away
            s = B.rn16_sat(B.rn32(max(abs(v) for v in xs) / (2 ** (bits - 1) - 1)))
            for j in range(1, 8):
                t = (Fraction(rng.randint(-5, 4)) + Fraction(1, 2)) * s
                t = B.rn32(t)
                ulp = Fraction(2) ** (B.floor_log2(abs(t)) - 23) if t else Fraction(0)
                xs[j] = t + rng.choice([-1, 0, 0, 1]) * ulp
        sb, codes = O.quant_block_int(np.array([float(v) for v in xs], np.float32), bits)
        s_ref, codes_ref = B.quant_block_int(xs, bits)
        assert Fraction(O.f16_to_f32(sb)) == s_ref
        assert list(codes) == codes_ref


def test_p9_brute_force_fp8_every_bf16_in_range():
    rng = random.Random(99)
    base = [B.bf16_exact(O.f32_to_bf16(rng.uniform(-3, 3))) for _ in range(32)]
    base[5] = Fraction(3)
    vals = bf16_values_in(-8, 8)[::3]                  # every third value keeps it quick
    for bits0 in vals:
        xs = list(base)
        xs[0] = B.bf16_exact(bits0)
        s_ref, codes_ref = B.quant_block_fp8(xs)
        s, codes = O.quant_block_fp8(np.array([float(v) for v in xs], np.float32))
        assert Fraction(s) == s_ref
        assert list(codes) == codes_ref


def test_p9_brute_force_fp8_fp32_extremes():
    """FP8 blocks of binary32 sums across the whole exponent range, including
    blocks whose scale a/448 falls below 2^-126 (flushed to a zero block)."""
    rng = random.Random(98)
    for i in range(1500):
        e = rng.randint(-150, 120)
        xs = [B.rn32(Fraction(rng.gauss(0, 1)) * Fraction(2) ** e) for _ in range(32)]
        s, codes = O.quant_block_fp8(np.array([float(v) for v in xs], np.float32))
        s_ref, codes_ref = B.quant_block_fp8(xs)
        assert Fraction(s) == s_ref
        assert list(codes) == codes_ref


def test_fp8_tiny_block_is_a_zero_block():
    # a/448 < 2^-126 for absmax 1e-36: the scale is flushed and every code is +0
    x = np.full(32, 1e-36, np.float32)
    x[3] = -1e-36
    s, codes = O.quant_block_fp8(x)
    assert s == 0.0 and all(codes == 0)


def test_negative_zero_inputs_sum_to_positive_zero():
    # the FP32 sum starts from +0.0f, so ranks that all send -0 still give +0
    nz = np.full(2048, 0x8000, np.uint16)
    for codec in ("fp8", "bf16", "int4", "int3"):
        outs, _ = O.allreduce([nz, nz], codec)
        assert np.all(outs[0] == 0)


def test_p9_e4m3_table_from_the_definition():
    for c in range(256):
        ref = B.e4m3_value(c)
        got = O.e4m3_to_f32(c)
        if ref is None:
            assert np.isnan(got) and (c & 0x7F) == 0x7F
        else:
            assert Fraction(got) == ref
    assert max(v for v, _ in B.E4M3_POS) == 448


def test_p9_binary16_conversion_brute_force():
    rng = random.Random(91)
    for _ in range(20000):
        x = f32(rng.choice([rng.gauss(0, 1) * 10.0 ** rng.uniform(-9, 5), rng.uniform(-70000, 70000)]))
        ref = B.round_binary(Fraction(x), 11, -14)
        got = O.f32_to_f16(x)
        if abs(ref) > 65504:
            assert (got & 0x7FFF) == 0x7C00
        else:
            assert Fraction(O.f16_to_f32(got)) == ref


# ---- P10: library special cases ---------------------------------------------
def _random_finite_f32(rng, k):
    u = rng.integers(0, 2 ** 32, size=k, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    return f[np.isfinite(f)]


def test_p10_binary16_matches_numpy():
    rng = np.random.default_rng(100)
    xs = np.concatenate([_random_finite_f32(rng, 60000),
                         (rng.standard_normal(60000) * 10.0 ** rng.uniform(-8, 5, 60000)).astype(np.float32)])
    with np.errstate(over="ignore"):                 # values above the f16 range become +-inf on both sides
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([O.f32_to_f16(x) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    h = np.arange(0x10000, dtype=np.uint16)
    h = h[(h & 0x7C00) != 0x7C00]
    back = np.array([O.f16_to_f32(v) for v in h], np.float32)
    assert np.array_equal(back, h.view(np.float16).astype(np.float32))


def test_p10_bfloat16_matches_torch():
    rng = np.random.default_rng(101)
    xs = np.concatenate([_random_finite_f32(rng, 60000),
                         (rng.standard_normal(60000) * 10.0 ** rng.uniform(-30, 30, 60000)).astype(np.float32)])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.f32_to_bf16(x) for x in xs], np.uint16)
    assert np.array_equal(got, ref)


def test_p10_e4m3_matches_torch_after_clamp():
    rng = np.random.default_rng(102)
    xs = np.concatenate([(rng.standard_normal(60000) * 10.0 ** rng.uniform(-5, 3, 60000)).astype(np.float32),
                         np.array([448, 464, 465, -1000, 2.0 ** -10, -(2.0 ** -10), 2.0 ** -12], np.float32)])
    clamped = np.clip(xs, -448, 448)
    ref = torch.from_numpy(clamped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.f32_to_e4m3(x) for x in xs], np.uint8)
    assert np.array_equal(got, ref)
    allc = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    mine = np.array([O.e4m3_to_f32(c) for c in range(256)], np.float32)
    assert np.array_equal(np.isnan(mine), np.isnan(allc))
    ok = ~np.isnan(allc)
    assert np.array_equal(mine[ok], allc[ok])


@pytest.mark.parametrize("N", [2, 3, 5])
def test_p10_bf16_passthrough_is_the_fp32_sum_in_rank_order(N):
    g = torch.Generator().manual_seed(103 + N)
    xs = [(torch.randn(8192, generator=g) * 10.0 ** (r - 2)).to(torch.bfloat16) for r in range(N)]
    acc = torch.zeros(8192, dtype=torch.float32)
    for x in xs:
        acc = acc + x.float()
    ref = acc.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    outs, used = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in xs], "bf16")
    assert used == "bf16"
    for o in outs:
        assert np.array_equal(o, ref)


def test_p10_rank_order_is_ascending():
    # 2^24 + 1 rounds back to 2^24 in binary32, so ((2^24 + 1) - 2^24) = 0 in rank
    # order, whereas any other order that pairs the large terms first gives 1.
    big, one = O.f32_to_bf16(2.0 ** 24), O.f32_to_bf16(1.0)
    nbig = O.f32_to_bf16(-(2.0 ** 24))
    ins = [np.full(2048, v, np.uint16) for v in (big, one, nbig)]
    outs, _ = O.allreduce(ins, "bf16")
    assert np.all(outs[0] == 0)
    ins = [np.full(2048, v, np.uint16) for v in (big, nbig, one)]
    outs, _ = O.allreduce(ins, "bf16")
    assert np.all(outs[0] == one)


# ---- P11: closed-form end-to-end bound --------------------------------------
def _exact_sum(ins):
    return sum(np.asarray(O.bf16_bits_to_f32(x), np.float64) for x in ins)


@pytest.mark.parametrize("codec,N", [("int4", 2), ("int3", 2), ("int4", 8), ("int3", 5), ("fp8", 2), ("fp8", 8)])
def test_p11_end_to_end_error_within_closed_form_bound(codec, N):
    g = torch.Generator().manual_seed(110 + N)
    n = 4096
    xs = [(torch.randn(n, generator=g) * 10.0 ** (0.5 * r - 1)).to(torch.bfloat16) for r in range(N)]
    ins = [x.view(torch.int16).numpy().view(np.uint16) for x in xs]
    outs, _ = O.allreduce(ins, codec)
    exact = _exact_sum(ins)
    out = O.bf16_bits_to_f32(outs[0]).astype(np.float64)
    # per-block quantities from the stage-1 wires and the gathered wire
    wires = [O.quantize(x, codec) for x in ins]
    gather = O.reduce(wires, 0, n // 2048, codec)
    v1 = [np.concatenate([O.dequant_tile(w[t * O.tile_bytes(codec):(t + 1) * O.tile_bytes(codec)], codec)
                          for t in range(n // 2048)]).astype(np.float64) for w in wires]
    v2 = np.concatenate([O.dequant_tile(gather[t * O.tile_bytes(codec):(t + 1) * O.tile_bytes(codec)], codec)
                         for t in range(n // 2048)]).astype(np.float64)
    x64 = [O.bf16_bits_to_f32(x).astype(np.float64) for x in ins]
    blk = np.arange(n) // 32
    if codec in ("int4", "int3"):
        qmax = 7 if codec == "int4" else 3
        s1 = [np.array([np.max(np.abs(v[b * 32:(b + 1) * 32])) / qmax for b in range(n // 32)])[blk] for v in v1]
        s2 = np.array([np.max(np.abs(v2[b * 32:(b + 1) * 32])) / qmax for b in range(n // 32)])[blk]
        stage1 = sum(s / 2 for s in s1)
        stage2 = s2 / 2
    else:
        def fp8_term(x, s):
            return np.abs(x) / 16 + s / 1024 + np.abs(x) * 2.0 ** -21
        s1 = [np.array([np.max(np.abs(x[b * 32:(b + 1) * 32])) / 448 for b in range(n // 32)])[blk] for x in x64]
        acc = np.sum(v1, axis=0)
        s2 = np.array([np.max(np.abs(acc[b * 32:(b + 1) * 32])) / 448 for b in range(n // 32)])[blk]
        stage1 = sum(fp8_term(x, s * (1 + 2.0 ** -20)) for x, s in zip(x64, s1))
        stage2 = fp8_term(acc, s2 * (1 + 2.0 ** -20))
    sum_err = (N - 1) * 2.0 ** -24 * np.sum(np.abs(v1), axis=0)
    bound = stage1 + sum_err + stage2 + 2.0 ** -8 * np.abs(v2)
    assert np.all(np.abs(out - exact) <= bound * (1 + 1e-12))


# ---- P12: every rank receives the same bits; threshold reading -----------------
@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "bf16"])
def test_p12_all_ranks_identical(codec):
    g = torch.Generator().manual_seed(120)
    xs = [torch.randn(6144, generator=g).to(torch.bfloat16) for _ in range(4)]
    outs, _ = O.allreduce([x.view(torch.int16).numpy().view(np.uint16) for x in xs], codec)
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_threshold_reading():
    F = facts()
    thr = F["int3_activation_threshold_bytes"]["value"]
    n = thr // 2                                          # exactly 1 MiB per rank
    x = np.zeros(n, np.uint16)
    _, used = O.allreduce([x, x], "int3", min_quant_bytes=thr)
    assert used == "int3"
    _, used = O.allreduce([x[:n - 2048], x[:n - 2048]], "int3", min_quant_bytes=thr)
    assert used == "bf16"


def test_shard_partition_does_not_change_values():
    g = torch.Generator().manual_seed(121)
    xs = [torch.randn(2048 * 7, generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
          for _ in range(3)]
    for codec in ("int4", "int3", "fp8", "bf16"):
        wires = [O.quantize(x, codec) if codec != "bf16" else x.view(np.uint8).copy() for x in xs]
        whole = O.reduce(wires, 0, 7, codec)
        pieces = np.zeros_like(whole)
        for t0, cnt in ((0, 2), (2, 1), (3, 4)):
            O.reduce(wires, t0, cnt, codec, pieces)
        assert np.array_equal(whole, pieces)
