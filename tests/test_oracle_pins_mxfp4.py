"""Pins of the oracle's MXFP4 codec (CPU only).

MXFP4 is the FP4 mode of the all-reduce: E2M1 elements ("Microscaling Data
Formats for Deep Learning", abstract: narrow floating-point elements sharing a
per-block scale; "QuickReduce INT3 Quantization and Benchmarking on MI355",
Summary: the INT4 and FP4 modes of the same all-reduce) with one power-of-two
E8M0 scale per 32 elements.  Nothing here re-types the oracle's formulas: the
checks use the E2M1 magnitude list, an exact-rational search (tests/brute.py),
torch's own E8M0 decoding, closed-form bounds and invariants.
"""
import random
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import brute as B

TWO = Fraction(2)


def f32_bits(x):
    return struct.unpack("<I", struct.pack("<f", x))[0]


def exact(x):
    return Fraction(float(np.float32(x)))


def neg(x):
    return bool(f32_bits(float(np.float32(x))) >> 31)


# ---- M1: sizes ---------------------------------------------------------------
def test_m1_tile_bytes():
    # 2048 four-bit elements plus 64 one-byte scales (one per 32 elements)
    assert O.tile_bytes("mxfp4") == 2048 * 4 // 8 + 64 == 1088
    assert O.wire_bytes("mxfp4", 2048 * 7) == 7 * 1088
    assert O.tile_bytes("mxfp4") < O.tile_bytes("int4")       # 1-byte scale instead of binary16


# ---- M2: the E2M1 element format -----------------------------------------------
def test_m2_e2m1_decode_table():
    for c in range(16):
        v = O.e2m1_to_f32(c)
        mag = B.E2M1_MAGNITUDES[c & 7]
        assert abs(Fraction(v)) == mag
        assert (struct.unpack("<I", struct.pack("<f", v))[0] >> 31) == (c >> 3)   # sign bit, -0 included


def test_m2_e2m1_encode_matches_nearest_search():
    # every multiple of 1/32 in [-9, 9] plus a few far values, both signs
    ys = [Fraction(k, 32) for k in range(-9 * 32, 9 * 32 + 1)] + [Fraction(10 ** 6), Fraction(-7, 1)]
    for y in ys:
        assert O.e2m1_rne(float(y)) == B.e2m1_rne_satfinite(y, y < 0), y
    # -0 keeps its sign bit; +0 does not
    assert O.e2m1_rne(-0.0) == 0x8 and O.e2m1_rne(0.0) == 0x0
    # each midpoint of the grid goes to the even mantissa
    assert [O.e2m1_rne(y) for y in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == [0, 2, 2, 4, 4, 6, 6]


# ---- M3: the E8M0 scale against torch's own decoding -------------------------------
def test_m3_e8m0_matches_torch():
    codes = torch.arange(0, 255, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).tolist()
    for c, r in zip(range(255), ref):
        assert O.e8m0_value(c) == r
        # dequantising the E2M1 value 1.0 (code 2) with scale code c gives 2^(c-127)
        if c >= 1:
            assert O.dequant_mxfp4(2, c) == r


# ---- M4: the shared exponent puts the absmax into [4, 8) -----------------------------
def test_m4_shared_exponent_bracket():
    rng = random.Random(7)
    for _ in range(3000):
        e = rng.randint(-140, 120)
        x = (np.float32(rng.uniform(-1, 1)) * np.float32(2.0) ** np.float32(e) * np.ones(32, np.float32)
             * np.array([rng.uniform(-1, 1) for _ in range(32)], np.float32))
        x = x.astype(np.float32)
        sc, _ = O.quant_block_mxfp4(x)
        a = max(abs(exact(v)) for v in x)
        assert sc - 127 == B.mx_shared_exponent(a)
        if a != 0 and sc > 0:
            assert 4 * TWO ** (sc - 127) <= a < 8 * TWO ** (sc - 127)


# ---- M5: brute force on tiny blocks (every BF16 value at one position) --------------
@pytest.mark.parametrize("others", [0.75, 3.0, 2.0 ** -126, 2.0 ** -133])
def test_m5_brute_force_single_position(others):
    rng = random.Random(11)
    base = np.array([others * rng.choice([-1, 1]) * rng.choice([1, 0.5, 0.25, 0]) for _ in range(32)], np.float32)
    for bits in range(0, 0x10000, 7):
        if (bits & 0x7F80) == 0x7F80:
            continue
        v = struct.unpack("<f", struct.pack("<I", bits << 16))[0]
        if abs(v) > 2.0 ** 100:
            continue
        x = base.copy()
        x[5] = v
        sc, codes = O.quant_block_mxfp4(x)
        E, ref = B.quant_block_mxfp4([exact(t) for t in x], [neg(t) for t in x])
        assert sc == E + 127
        assert list(codes) == ref, (v, sc)


# ---- M6: on-grid values round-trip exactly ------------------------------------------
def test_m6_on_grid_round_trip():
    rng = random.Random(3)
    for _ in range(400):
        E = rng.randint(-127, 120)
        k = [rng.choice(B.E2M1_MAGNITUDES) * rng.choice([-1, 1]) for _ in range(32)]
        k[rng.randrange(32)] = rng.choice([Fraction(4), Fraction(6)]) * rng.choice([-1, 1])
        x = np.array([float(v * TWO ** E) for v in k], np.float32)
        sc, codes = O.quant_block_mxfp4(x)
        assert sc == E + 127
        for c, v in zip(codes, x):
            assert O.dequant_mxfp4(c, sc) == v


# ---- M7: zero blocks ------------------------------------------------------------------
def test_m7_zero_block():
    sc, codes = O.quant_block_mxfp4(np.zeros(32, np.float32))
    assert sc == 0 and list(codes) == [0] * 32
    x = np.zeros(32, np.float32)
    x[::2] = -0.0
    sc, codes = O.quant_block_mxfp4(x)
    assert sc == 0 and list(codes) == [8, 0] * 16
    assert f32_bits(O.dequant_mxfp4(8, 0)) == 0x80000000


# ---- M8: error of one stage -------------------------------------------------------------
def test_m8_stage_error_bound():
    rng = np.random.default_rng(5)
    for _ in range(300):
        x = (rng.standard_t(3, 32) * 2.0 ** rng.integers(-30, 30)).astype(np.float32)
        sc, codes = O.quant_block_mxfp4(x)
        E = sc - 127
        for c, xv in zip(codes, x):
            err = abs(exact(xv) - Fraction(O.dequant_mxfp4(c, sc)))
            y = abs(exact(xv)) / TWO ** E
            # half a grid step below 6 (0.25 below 2, 0.5 below 4, 1 up to 6),
            # the saturation distance above it
            bound = (y - 6 if y > 6 else (Fraction(1, 4) if y < 2 else Fraction(1, 2) if y < 4 else 1)) * TWO ** E
            assert err <= bound


# ---- M9: idempotence, so the N = 1 all-reduce is one round trip --------------------------
def test_m9_idempotent_and_n1():
    rng = np.random.default_rng(9)
    for _ in range(200):
        x = (rng.standard_normal(2048) * 2.0 ** rng.integers(-20, 20)).astype(np.float32)
        t = O.quant_tile(x, "mxfp4")
        assert np.array_equal(O.quant_tile(O.dequant_tile(t, "mxfp4"), "mxfp4"), t)
    xb = torch.randn(2048 * 3, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    outs, used = O.allreduce([bits], "mxfp4")
    assert used == "mxfp4"
    one_trip = O.decode(O.quantize(bits, "mxfp4"), bits.size, "mxfp4")
    # equal as values; a negative zero of the round trip becomes +0 in the
    # all-reduce, whose FP32 sum starts from +0 (+0 + -0 = +0)
    same = (outs[0] == one_trip) | ((one_trip == 0x8000) & (outs[0] == 0))
    assert np.all(same) and np.any(one_trip == 0x8000)


# ---- M10: antisymmetric inputs sum to exactly +0 -----------------------------------------
def test_m10_antisymmetry():
    x = torch.randn(2048 * 2, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    a = x.view(torch.int16).numpy().view(np.uint16)
    b = (-x).view(torch.int16).numpy().view(np.uint16)
    outs, _ = O.allreduce([a, b], "mxfp4")
    for o in outs:
        assert np.all(o == 0)


# ---- M11: closed-form end-to-end bound, identical outputs --------------------------------
def test_m11_end_to_end_bound():
    N, n = 4, 2048 * 2
    g = torch.Generator().manual_seed(3)
    xs = [torch.randn(n, generator=g).to(torch.bfloat16) for _ in range(N)]
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in xs]
    outs, _ = O.allreduce(bits, "mxfp4")
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    wires = [O.quantize(b, "mxfp4") for b in bits]
    out = O.bf16_bits_to_f32(outs[0]).astype(np.float64)
    exact_sum = sum(x.double().numpy() for x in xs)
    for t in range(n // 2048):
        v = [O.dequant_tile(w[t * 1088:(t + 1) * 1088], "mxfp4").astype(np.float64) for w in wires]
        for blk in range(64):
            sl = slice(t * 2048 + blk * 32, t * 2048 + blk * 32 + 32)
            ls = slice(blk * 32, blk * 32 + 32)
            # stage 1: at most 2^(E+1) per rank (the saturation case); FP32 sum:
            # (N-1) half-ulps of the running sums; stage 2 likewise; BF16: 2^-8 relative
            s1 = sum(2.0 ** (int(w[t * 1088 + 1024 + blk]) - 127 + 1) for w in wires)
            fp32 = (N - 1) * 2.0 ** -24 * sum(np.abs(vr[ls]) for vr in v)
            acc = sum(vr[ls] for vr in v)
            E2 = B.mx_shared_exponent(Fraction(float(np.max(np.abs(acc))))) if np.any(acc) else -127
            bound = s1 + fp32 + 2.0 ** (E2 + 1) + 2.0 ** -8 * np.abs(out[sl])
            assert np.all(np.abs(out[sl] - exact_sum[sl]) <= bound + 1e-300)
