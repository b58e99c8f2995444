"""Byte-level pins of the oracle's tile layouts (CPU only).

"QuickReduce INT3 Quantization and Benchmarking on MI355", Summary, prints the
transmitted tile sizes (1152 B for INT4, 896 B for INT3).  Those counts fit only
2048 packed codes followed by 64 binary16 block scales; where inside the tile
each code and scale sits is a reading, the same for every codec:

* codes first, in element order; INT4 and MXFP4 put element 2k in the LOW
  nibble of byte k and element 2k+1 in the high nibble;
* the per-block scales last, one per 32-element block in block order, at byte
  1024 (INT4 binary16, MXFP4 E8M0), 768 (INT3, after the q2w and q1w planes)
  or 2048 (FP8 binary32), multi-byte scales little-endian;
* the BF16 passthrough tile is the 2048 binary16 words in element order,
  little-endian.

Every expected byte below is derived by hand in the comment beside it from the
format definitions ("FP8 Formats for Deep Learning" for E4M3, "Microscaling
Data Formats for Deep Learning" for E2M1 and E8M0, IEEE 754 for binary16 and
binary32), not by calling the oracle.  Each codec is pinned from both sides:
the quantiser's bytes (pack), and the values decoded from tile bytes the test
writes itself (unpack), so a layout change made the same way on both sides of
the oracle still fails here.  INT3's own worked tile is in test_oracle_pins.py.
"""
import struct

import numpy as np

from oracle import oracle as O


def le16(v):
    return [v & 0xFF, v >> 8]


def le32_of_f32(x):
    return list(struct.pack("<f", x))


# ---- INT4: 1024 B of nibbles, then 64 binary16 scales at byte 1024 --------------
def test_int4_worked_tile_bytes():
    x = np.zeros(2048, np.float32)
    # block 0: absmax 7 -> s = fl32(7/7) = 1.0, binary16 0x3C00.  q = RNE(x):
    # 7 -> 7, -3.5 -> -4 (tie to even), 1.75 -> 2, 0.5 -> 0 (tie), 1.5 -> 2,
    # 2.5 -> 2 (tie), -2.5 -> -2, 6.5 -> 6 (tie), -7 -> -7; codes q + 8 =
    # 15, 4, 10, 8, 10, 10, 6, 14, 1, and 8 for the 23 zeros.
    x[:9] = [7, -3.5, 1.75, 0.5, 1.5, 2.5, -2.5, 6.5, -7]
    # block 1: only element 33 = 1.0.  s = f16(fl32(1/7)): 1/7 = 2^-3 * 1.142857..,
    # 0.142857 * 1024 = 146.3 -> 146, so binary16 (12 << 10) | 146 = 0x3092.
    # 1/s = 7.0017 -> q = 7, code 15; element 32 = 0 -> code 8.
    x[33] = 1.0
    # block 63: only element 2047 = -14 -> s = 2.0 (0x4000), q = -7, code 1.
    x[2047] = -14.0
    tile = O.quant_tile(x, "int4")
    assert tile.size == 1152
    # element 2k in the low nibble: (15 | 4<<4), (10 | 8<<4), (10 | 10<<4), (6 | 14<<4), (1 | 8<<4)
    assert list(tile[0:5]) == [0x4F, 0x8A, 0xAA, 0xE6, 0x81]
    assert all(tile[5:16] == 0x88)                  # code 8 (q = 0) in both nibbles
    assert tile[16] == 0xF8                         # element 32 code 8 low, element 33 code 15 high
    assert all(tile[17:1023] == 0x88)               # all-zero blocks: q = 0 everywhere
    assert tile[1023] == 0x18                       # element 2046 code 8 low, element 2047 code 1 high
    # scales at byte 1024 + 2b, little-endian; all-zero blocks have scale +0
    assert list(tile[1024:1026]) == le16(0x3C00) == [0x00, 0x3C]
    assert list(tile[1026:1028]) == le16(0x3092) == [0x92, 0x30]
    assert all(tile[1028:1150] == 0)
    assert list(tile[1150:1152]) == le16(0x4000) == [0x00, 0x40]
    assert [O.tile_codes(tile, "int4")[i] for i in (0, 1, 32, 33, 2046, 2047)] == [15, 4, 8, 15, 8, 1]


def test_int4_decode_of_hand_written_tile():
    tile = np.full(1152, 0x88, np.uint8)            # every code 8 (q = 0) ...
    tile[1024:] = 0                                 # ... and every scale +0
    tile[0] = 0x1F                                  # element 0 code 15 (q = +7), element 1 code 1 (q = -7)
    tile[1024:1026] = [0x00, 0x40]                  # block 0 scale 0x4000 = 2.0
    tile[32] = 0x89                                 # element 64 (block 2) code 9: q = +1; element 65 q = 0
    tile[1028:1030] = [0x92, 0x30]                  # block 2 scale 0x3092 = 1170/8192
    tile[1151] = 0x3C                               # block 63 scale 0x3C00 = 1.0 (high byte at 1151)
    tile[1023] = 0x08 | (0xC << 4)                  # element 2047 code 12: q = +4
    v = O.dequant_tile(tile, "int4")
    expect = np.zeros(2048, np.float32)
    expect[0], expect[1] = 14.0, -14.0
    expect[64] = 1170 / 8192
    expect[2047] = 4.0
    assert np.array_equal(v, expect)


# ---- FP8: 2048 E4M3 codes, then 64 binary32 scales at byte 2048 ------------------
def test_fp8_worked_tile_bytes():
    x = np.zeros(2048, np.float32)
    # block 0: absmax 448 -> s = 448/448 = 1.0, so the codes are the E4M3 values of
    # the inputs: 448 = 0x7E (max finite), 1 = 0x38, 17 ties 16/18 -> 16 = 0x58,
    # -2^-9 = subnormal 1 with sign = 0x81, 2^-10 ties 0/2^-9 -> 0x00,
    # 3*2^-11 is nearest 2^-9 = 0x01, -300 lies between 288 and 320 -> -288 = 0xF9.
    x[:7] = [448, 1.0, 17.0, -2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, -300]
    # block 2: element 69 = -896 -> s = 2.0 exactly, 1/s = 0.5, y = -448 -> 0xFE.
    x[69] = -896.0
    # block 63: element 2047 = 1.0 -> s = fl32(1/448): 1/448 = 2^-9 * 1.142857..,
    # mantissa 0.142857 * 2^23 = 1198372.57 -> 1198373 = 0x124925, exponent
    # 118 -> bits 0x3B124925.  fl32(1/s) lies within an ulp of 448 and every value
    # above 432 encodes (RNE, satfinite) to 448 = 0x7E.
    x[2047] = 1.0
    tile = O.quant_tile(x, "fp8")
    assert tile.size == 2304
    assert list(tile[0:7]) == [0x7E, 0x38, 0x58, 0x81, 0x00, 0x01, 0xF9]
    assert all(tile[7:69] == 0) and tile[69] == 0xFE and all(tile[70:2047] == 0)
    assert tile[2047] == 0x7E
    # binary32 scales at byte 2048 + 4b, little-endian
    assert list(tile[2048:2052]) == [0x00, 0x00, 0x80, 0x3F]       # 1.0 = 0x3F800000
    assert all(tile[2052:2056] == 0)                                 # block 1: all zero -> +0
    assert list(tile[2056:2060]) == [0x00, 0x00, 0x00, 0x40]       # 2.0 = 0x40000000
    assert all(tile[2060:2300] == 0)
    assert list(tile[2300:2304]) == [0x25, 0x49, 0x12, 0x3B]       # 0x3B124925
    # the hand-derived bits are the IEEE quotient (numpy divides with one rounding)
    assert le32_of_f32(np.float32(1) / np.float32(448)) == [0x25, 0x49, 0x12, 0x3B]


def test_fp8_decode_of_hand_written_tile():
    tile = np.zeros(2304, np.uint8)
    tile[0] = 0x38                                   # 1.0
    tile[31] = 0xC0                                  # -2.0
    tile[2048:2052] = le32_of_f32(0.25)              # block 0 scale 0.25 = 0x3E800000
    tile[2047] = 0x7E                                # 448
    tile[2300:2304] = [0x00, 0x00, 0x00, 0x40]       # block 63 scale 2.0
    v = O.dequant_tile(tile, "fp8")
    expect = np.zeros(2048, np.float32)
    expect[0], expect[31], expect[2047] = 0.25, -0.5, 896.0
    assert np.array_equal(v, expect)


# ---- MXFP4: 1024 B of E2M1 nibbles, then 64 E8M0 scale bytes at byte 1024 -------
# E2M1 code = sign<<3 | e<<1 | m; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7.
# E8M0 byte = E + 127 with E = floor(log2 absmax) - 2 (2 = E2M1's largest exponent).
def test_mxfp4_worked_tile_bytes():
    x = np.zeros(2048, np.float32)
    # block 0: absmax 6 = 1.5 * 2^2 -> E = 0, byte 0x7F; x / 1:
    # 6 -> 7, -0.5 -> 8|1 = 9, 1.5 -> 3, -4 -> 8|6 = 14, 3 -> 5,
    # 2.5 ties 2 (m = 0) and 3 (m = 1) -> 2, code 4 (even mantissa).
    x[:6] = [6, -0.5, 1.5, -4, 3, 2.5]
    # block 7: absmax 0.75 = 1.5 * 2^-1 -> E = -3, byte 124 = 0x7C;
    # element 226 = -0.0625 -> -0.5 -> code 9; element 227 = 0.75 -> 6 -> code 7.
    x[226], x[227] = -0.0625, 0.75
    # block 63: absmax 1000 = 1.95 * 2^9 -> E = 7, byte 134 = 0x86;
    # 1000 / 128 = 7.8125 saturates to 6 -> code 7, element 2046 (low nibble).
    x[2046] = 1000.0
    tile = O.quant_tile(x, "mxfp4")
    assert tile.size == 1088
    assert list(tile[0:3]) == [0x97, 0xE3, 0x45]    # (7 | 9<<4), (3 | 14<<4), (5 | 4<<4)
    assert all(tile[3:113] == 0)                    # +0 codes, all-zero blocks included
    assert tile[113] == 0x79                        # element 226 low nibble 9, element 227 high nibble 7
    assert all(tile[114:1023] == 0)
    assert tile[1023] == 0x07
    # one scale byte per block at 1024 + b; an all-zero block has E = -127, byte 0
    assert tile[1024] == 0x7F and tile[1031] == 0x7C and tile[1087] == 0x86
    assert all(tile[1025:1031] == 0) and all(tile[1032:1087] == 0)


def test_mxfp4_decode_of_hand_written_tile():
    tile = np.zeros(1088, np.uint8)
    tile[0] = 0x9E                                   # element 0 code 14 (-4), element 1 code 9 (-0.5)
    tile[1024] = 0x80                                # block 0: E = 1, scale 2
    tile[1023] = 0x70                                # element 2047 code 7 (6)
    tile[1087] = 0x7D                                # block 63: E = -2, scale 1/4
    v = O.dequant_tile(tile, "mxfp4")
    expect = np.zeros(2048, np.float32)
    expect[0], expect[1], expect[2047] = -8.0, -1.0, 1.5
    assert np.array_equal(v, expect)


# ---- BF16 passthrough: 2048 little-endian binary16 words ------------------------
def test_bf16_tile_bytes_and_decode():
    x = np.zeros(2048, np.float32)
    x[0], x[1], x[2047] = 1.0, -2.5, 3.0             # BF16 0x3F80, 0xC020, 0x4040
    tile = O.quant_tile(x, "bf16")
    assert tile.size == 4096
    assert list(tile[0:4]) == [0x80, 0x3F, 0x20, 0xC0]
    assert list(tile[4094:4096]) == [0x40, 0x40] and all(tile[4:4094] == 0)
    hand = np.zeros(4096, np.uint8)
    hand[2:4] = [0xC0, 0x3F]                         # element 1 = 0x3FC0 = 1.5
    v = O.dequant_tile(hand, "bf16")
    assert v[1] == 1.5 and np.count_nonzero(v) == 1


# ---- INT3: decode of a hand-written tile (its pack side is pinned elsewhere) ----
def test_int3_decode_of_hand_written_tile():
    tile = np.zeros(896, np.uint8)
    # element i: low two bits at bits 2(i%4) of byte i/4, high bit at bit i%8 of
    # byte 512 + i/8; scales at 768 + 2b.  Elements 0..3 codes 7, 1, 4, 0 -> q
    # = +3, -3, 0, -4; the last code (0) is outside the symmetric range but still
    # decodes by the offset: q = code - 4.
    tile[0] = 0b00_00_01_11                          # low bits 3, 1, 0, 0
    tile[512] = 0b0000_0101                          # high bits 1, 0, 1, 0
    tile[768:770] = [0x00, 0x3C]                     # block 0 scale 1.0
    # every other element: code 0 low bits and high bit 0 -> q = -4, times scale 0 -> 0
    v = O.dequant_tile(tile, "int3")
    assert list(v[:4]) == [3.0, -3.0, 0.0, -4.0]
    assert np.count_nonzero(v[4:32]) == 28 and all(v[4:32] == -4.0)
    assert np.count_nonzero(v[32:]) == 0
