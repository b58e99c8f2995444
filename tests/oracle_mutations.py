"""Plausible mistakes planted in copies of the CPU oracle (test data only).

Each entry is (name, [(old, new), ...]): every `old` text of
``oracle/lpar_oracle.c`` is replaced by `new` (first occurrence), the copy is
compiled, and the named pin files must then fail.  The lists cover the block
quantisers, the number formats, the tile layouts, the reduction order, the
threshold, the collectives and the binary32 path.

LAYOUT holds layout changes made the same way on the packing and on the
unpacking side.  The round trip through such an oracle is still exact, so only
the byte-level worked tiles (hand-derived bytes, and hand-written tiles
decoded) can catch them.
"""

# core: caught by test_oracle_pins.py
CORE = [
    ('absmax uses min',
     [('if (m > a) a = m;\n    }\n    float ratio',
       'if (m < a || j == 0) a = m;\n    }\n    float ratio')]),
    ('ratio divides by qmax+1',
     [('a / (float)qmax',
       'a / (float)(qmax + 1)')]),
    ('no f16 saturation',
     [('if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFF;',
       '')]),
    ('ties away from zero',
     [('double qd = nearbyint((double)x[j] / (double)s);',
       'double qd = round((double)x[j] / (double)s);')]),
    ('no upper clamp',
     [('if (qd > qmax) qd = qmax;',
       '')]),
    ('no lower clamp',
     [('if (qd < -qmax) qd = -qmax;',
       '')]),
    ('bias off by one',
     [('codes[j] = (uint8_t)(q + bias);',
       'codes[j] = (uint8_t)(q + bias - 1);')]),
    ('int4 nibble order',
     [('tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));\n            }\n            put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);',
       'tile[i / 2] |= (uint8_t)(codes[j] << (4 * (1 - i % 2)));\n            }\n            put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);')]),
    ('int3 planes swapped',
     [('uint8_t *q2w = tile;\n            uint8_t *q1w = tile + ORC_TILE_ELEMS / 4;',
       'uint8_t *q1w = tile;\n            uint8_t *q2w = tile + ORC_TILE_ELEMS / 8;')]),
    ('int3 q2w bit order',
     [('q2w[i / 4] |= (uint8_t)((codes[j] & 3) << (2 * (i % 4)));',
       'q2w[i / 4] |= (uint8_t)((codes[j] & 3) << (6 - 2 * (i % 4)));')]),
    ('int4 scale offset',
     [('put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);',
       'put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * ((b + 1) % 64), sb);')]),
    ('fp8 max 240',
     [('float s = a / 448.0f;',
       'float s = a / 240.0f;')]),
    ('fp8 divide instead of reciprocal',
     [('float y = x[j] * inv;',
       'float y = x[j] / s; (void)inv;')]),
    ('fp8 no flush of tiny scale',
     [('if (s < 0x1p-126f) {',
       'if (s == 0.0f) {')]),
    ('fp8 dequant adds',
     [('return orc_e4m3_to_f32(code) * scale;',
       'return orc_e4m3_to_f32(code) * scale + 0.0f * scale + (code == 0x38 ? scale * 0x1p-20f : 0.0f);')]),
    ('reverse rank order',
     [('for (int r = 0; r < N; ++r) {\n            orc_dequant_tile',
       'for (int r = N - 1; r >= 0; --r) {\n            orc_dequant_tile')]),
    ('drop last rank',
     [('for (int r = 0; r < N; ++r) {\n            orc_dequant_tile',
       'for (int r = 0; r < N - (N > 2); ++r) {\n            orc_dequant_tile')]),
    ('bf16 truncates',
     [('double r = round_to_format(fabs((double)x), 8, -126);',
       'double r = floor(fabs((double)x) / ldexp(1.0, (int)floor(log2(fabs((double)x))) - 7)) * ldexp(1.0, (int)floor(log2(fabs((double)x))) - 7); if (x == 0) r = 0;')]),
    ('f16 emin -15',
     [('round_to_format(fabs((double)x), 11, -14)',
       'round_to_format(fabs((double)x), 11, -15)')]),
    ('e4m3 bias 8',
     [('else         v = ldexp(1.0 + (double)mf / 8.0, ef - 7);',
       'else         v = ldexp(1.0 + (double)mf / 8.0, ef - 8);')]),
    ('int dequant off by one',
     [('int q = (int)code - (1 << (bits - 1));',
       'int q = (int)code - (1 << (bits - 1)) + (code > 12);')]),
    ('threshold <=',
     [('2 * n < min_quant_bytes',
       '2 * n <= min_quant_bytes')]),
    ('reduce writes compact',
     [('orc_quant_tile(acc, codec, wire_out + t * tb);',
       'orc_quant_tile(acc, codec, wire_out + (t - tile_begin) * tb);')]),
    ('acc starts from first term',
     [('for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = +0.0f;',
       'for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = -0.0f;')]),
    ('int3 q1w bit order',
     [('q1w[i / 8] |= (uint8_t)((codes[j] >> 2) << (i % 8));',
       'q1w[i / 8] |= (uint8_t)((codes[j] >> 2) << (7 - i % 8));')]),
    ('int scale skips f16 rounding',
     [('float s = orc_f16_to_f32(sb);\n\n    for',
       'float s = ratio > 65504.0f ? 65504.0f : ratio;\n\n    for')]),
    ('fp8 scale position',
     [('put_f32_le(tile + ORC_TILE_ELEMS + 4 * b, s);',
       'put_f32_le(tile + ORC_TILE_ELEMS + 4 * (63 - b), s);')]),
    ('bf16 decode of gather truncated',
     [('out_bf16[t * ORC_TILE_ELEMS + i] = orc_f32_to_bf16_rne(v[i]);',
       '{ uint32_t u; memcpy(&u, &v[i], 4); out_bf16[t * ORC_TILE_ELEMS + i] = (uint16_t)(u >> 16); }')]),
    ('e4m3 encode no subnormal grid',
     [('double r = isinf(x) ? 448.0 : round_to_format(a, 4, -6);',
       'double r = isinf(x) ? 448.0 : round_to_format(a, 4, -9);')]),
]

# mxfp4: caught by test_oracle_pins_mxfp4.py
MXFP4 = [
    ('mx offset -1',
     [('E = (F - 1) - 2;',
       'E = (F - 1) - 1;')]),
    ('mx ceil log2',
     [('E = (F - 1) - 2;',
       'E = F - 2;')]),
    ('mx clamp -126',
     [('if (E < -127) E = -127;',
       'if (E < -126) E = -126;')]),
    ('mx no low clamp',
     [('if (E < -127) E = -127;',
       '')]),
    ('mx zero block scale 127',
     [('int E = -127;\n    if (a > 0.0f)',
       'int E = 0;\n    if (a > 0.0f)')]),
    ('mx scale code bias 128',
     [('*scale_code = (uint8_t)(E + 127);',
       '*scale_code = (uint8_t)(E + 128);')]),
    ('e2m1 ties away',
     [('double r = round_to_format(fabs(y), 2, 0);',
       'double r = fabs(y) < 2 ? round(fabs(y) * 2) / 2 : fabs(y) < 4 ? round(fabs(y)) : round(fabs(y) / 2) * 2;')]),
    ('e2m1 no saturation',
     [('if (r > 6.0) r = 6.0;',
       'if (r > 8.0) r = 8.0;')]),
    ('e2m1 sign dropped on zero',
     [('uint8_t sign = signbit(y) ? 0x8 : 0x0;',
       'uint8_t sign = (y < 0) ? 0x8 : 0x0;')]),
    ('e2m1 subnormal grid',
     [('double r = round_to_format(fabs(y), 2, 0);',
       'double r = round_to_format(fabs(y), 2, -1);')]),
    ('e2m1 decode bias 2',
     [('double v = (ef == 0) ? 0.5 * mf : ldexp(1.0 + 0.5 * mf, ef - 1);',
       'double v = (ef == 0) ? 0.5 * mf : ldexp(1.0 + 0.5 * mf, ef - 2);')]),
    ('mx nibble order',
     [('tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));\n            }\n            tile[ORC_TILE_ELEMS / 2 + b] = sc;',
       'tile[i / 2] |= (uint8_t)(codes[j] << (4 * (1 - i % 2)));\n            }\n            tile[ORC_TILE_ELEMS / 2 + b] = sc;')]),
    ('mx scale position',
     [('tile[ORC_TILE_ELEMS / 2 + b] = sc;',
       'tile[ORC_TILE_ELEMS / 2 + (63 - b)] = sc;')]),
    ('mx dequant uses E+1',
     [('orc_e8m0_to_f64(scale_code));',
       'orc_e8m0_to_f64(scale_code + 1));')]),
    ('mx scales by multiply 2^E',
     [('ldexp((double)x[j], -E)',
       'ldexp((double)x[j], E)')]),
]

# collectives: caught by test_oracle_pins_collectives.py
COLLECTIVES = [
    ('rs ceil partition',
     [('size_t t0 = (size_t)j * T / (size_t)N, t1 = (size_t)(j + 1) * T / (size_t)N;\n        for (size_t t = t0; t < t1; ++t)\n            reduce_tile_to_bf16',
       'size_t t0 = ((size_t)j * T + N - 1) / (size_t)N, t1 = ((size_t)(j + 1) * T + N - 1) / (size_t)N;\n        for (size_t t = t0; t < t1; ++t)\n            reduce_tile_to_bf16')]),
    ('rs shard reversed',
     [('reduce_tile_to_bf16(wires, N, t, codec, out_bf16[j] + (t - t0) * ORC_TILE_ELEMS);',
       'reduce_tile_to_bf16(wires, N, t, codec, out_bf16[j] + (t1 - 1 - t) * ORC_TILE_ELEMS);')]),
    ('reduce reverse order',
     [('    for (int r = 0; r < N; ++r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]',
       '    for (int r = N - 1; r >= 0; --r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]')]),
    ('reduce drops last rank',
     [('    for (int r = 0; r < N; ++r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]',
       '    for (int r = 0; r < N - (N > 1); ++r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]')]),
    ('oneshot requantises',
     [('    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i] = orc_f32_to_bf16_rne(acc[i]);',
       '    if (codec != ORC_BF16) { uint8_t tmp[4096]; orc_quant_tile(acc, codec, tmp); orc_dequant_tile(tmp, codec, acc); }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i] = orc_f32_to_bf16_rne(acc[i]);')]),
    ('ag destination by receiver',
     [('else orc_decode(wires[r], m, codec, out_bf16[j] + (size_t)r * m);',
       'else orc_decode(wires[r], m, codec, out_bf16[j] + (size_t)((r + j) % N) * m);')]),
    ('a2a wrong segment',
     [('const uint8_t *seg = wires[r] + (size_t)j * seg_wire;',
       'const uint8_t *seg = wires[r] + (size_t)r * seg_wire;')]),
    ('a2a threshold per segment',
     [('    size_t n = (size_t)N * m;\n    codec = effective(codec, 2 * n, min_quant_bytes);',
       '    size_t n = (size_t)N * m;\n    codec = effective(codec, 2 * m, min_quant_bytes);')]),
    ('ag threshold whole output',
     [('codec = effective(codec, 2 * m, min_quant_bytes);\n    uint8_t *wires[ORC_MAX_RANKS];\n    if (quantize_all(in_bf16, N, m,',
       'codec = effective(codec, 2 * m * N, min_quant_bytes);\n    uint8_t *wires[ORC_MAX_RANKS];\n    if (quantize_all(in_bf16, N, m,')]),
    ('bf16 sum truncated',
     [('    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i] = orc_f32_to_bf16_rne(acc[i]);',
       '    for (int i = 0; i < ORC_TILE_ELEMS; ++i) { uint32_t u; memcpy(&u, &acc[i], 4); dst[i] = (uint16_t)(u >> 16); }')]),
    ('acc starts -0',
     [('    for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = +0.0f;\n    for (int r = 0; r < N; ++r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]',
       '    for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = -0.0f;\n    for (int r = 0; r < N; ++r) {\n        orc_dequant_tile(wires[r] + t * tb, codec, v);\n        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];\n    }\n    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i]')]),
]

# f32: caught by test_oracle_pins_f32.py
F32 = [
    ('passthrough reversed',
     [('for (int r = 0; r < N; ++r) acc = acc + in_f32[r][i];',
       'for (int r = N - 1; r >= 0; --r) acc = acc + in_f32[r][i];')]),
    ('threshold on 2n',
     [('codec = effective(codec, 4 * n, min_quant_bytes);\n    size_t tiles = n / ORC_TILE_ELEMS;\n    if (codec == ORC_BF16) {',
       'codec = effective(codec, 2 * n, min_quant_bytes);\n    size_t tiles = n / ORC_TILE_ELEMS;\n    if (codec == ORC_BF16) {')]),
    ('output rounded to bf16',
     [('for (int r = 0; r < N; ++r) orc_dequant_tile(gather + t * tb, codec, out_f32[r] + t * ORC_TILE_ELEMS);',
       'for (int r = 0; r < N; ++r) { orc_dequant_tile(gather + t * tb, codec, out_f32[r] + t * ORC_TILE_ELEMS); for (int i = 0; i < ORC_TILE_ELEMS; ++i) out_f32[r][t * ORC_TILE_ELEMS + i] = orc_bf16_to_f32(orc_f32_to_bf16_rne(out_f32[r][t * ORC_TILE_ELEMS + i])); }')]),
    ('no requantisation',
     [('        orc_reduce((const uint8_t *const *)wires, N, t0, t1 - t0, codec, gather);\n    }\n    for (size_t t = 0; t < tiles; ++t)            /* all-gather',
       '        orc_reduce((const uint8_t *const *)wires, N, t0, t1 - t0, codec, gather);\n    }\n    if (N > 1) memcpy(gather, wires[0], wb);\n    for (size_t t = 0; t < tiles; ++t)            /* all-gather')]),
]

_NIBBLE_UNPACK = "case ORC_INT4:\n    case ORC_MXFP4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);"
_INT4_PACK = ("tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));\n            }\n"
              "            put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);")
_MX_PACK = ("tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));\n            }\n"
            "            tile[ORC_TILE_ELEMS / 2 + b] = sc;")
_INT4_SCALE_GET = "get_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b));"
_INT3_SCALE_PUT = "put_u16_le(tile + ORC_TILE_ELEMS / 4 + ORC_TILE_ELEMS / 8 + 2 * b, sb);"
_INT3_SCALE_GET = "get_u16_le(tile + ORC_TILE_ELEMS / 4 + ORC_TILE_ELEMS / 8 + 2 * b));"
_INT3_UNPACK = ("uint8_t lo = (uint8_t)((tile[i / 4] >> (2 * (i % 4))) & 3);\n"
                "        uint8_t hi = (uint8_t)((tile[ORC_TILE_ELEMS / 4 + i / 8] >> (i % 8)) & 1);")


def _swap16(e):
    return "(uint16_t)((%s >> 8) | (%s << 8))" % (e, e)


# layout: caught by test_oracle_pins_layout.py (INT3 also by test_oracle_pins.py)
LAYOUT = [
    ("int4 nibble order, pack and unpack",
     [(_INT4_PACK, _INT4_PACK.replace("(4 * (i % 2))", "(4 * (1 - i % 2))")),
      (_NIBBLE_UNPACK,
       "case ORC_INT4: return (uint8_t)((tile[i / 2] >> (4 * (1 - i % 2))) & 0xF);\n"
       "    case ORC_MXFP4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);")]),
    ("mxfp4 nibble order, pack and unpack",
     [(_MX_PACK, _MX_PACK.replace("(4 * (i % 2))", "(4 * (1 - i % 2))")),
      (_NIBBLE_UNPACK,
       "case ORC_INT4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);\n"
       "    case ORC_MXFP4: return (uint8_t)((tile[i / 2] >> (4 * (1 - i % 2))) & 0xF);")]),
    ("int4 scales in reverse block order, pack and unpack",
     [("put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);",
       "put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * (63 - b), sb);"),
      (_INT4_SCALE_GET, "get_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * (63 - b)));")]),
    ("int4 scales big-endian, pack and unpack",
     [("put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);",
       "put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, %s);" % _swap16("sb")),
      (_INT4_SCALE_GET, _swap16("get_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b)") + ");")]),
    ("int4 scales first, codes after them, pack and unpack",
     [(_INT4_PACK, _INT4_PACK.replace("tile[i / 2]", "tile[128 + i / 2]")
                             .replace("tile + ORC_TILE_ELEMS / 2 + 2 * b", "tile + 2 * b")),
      (_NIBBLE_UNPACK,
       "case ORC_INT4: return (uint8_t)((tile[128 + i / 2] >> (4 * (i % 2))) & 0xF);\n"
       "    case ORC_MXFP4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);"),
      (_INT4_SCALE_GET, "get_u16_le(tile + 2 * b));")]),
    ("fp8 scales big-endian, pack and unpack",
     [("p[0] = (uint8_t)u; p[1] = (uint8_t)(u >> 8); p[2] = (uint8_t)(u >> 16); p[3] = (uint8_t)(u >> 24);",
       "p[3] = (uint8_t)u; p[2] = (uint8_t)(u >> 8); p[1] = (uint8_t)(u >> 16); p[0] = (uint8_t)(u >> 24);"),
      ("(uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24)",
       "(uint32_t)p[3] | ((uint32_t)p[2] << 8) | ((uint32_t)p[1] << 16) | ((uint32_t)p[0] << 24)")]),
    ("fp8 scales in reverse block order, pack and unpack",
     [("put_f32_le(tile + ORC_TILE_ELEMS + 4 * b, s);", "put_f32_le(tile + ORC_TILE_ELEMS + 4 * (63 - b), s);"),
      ("get_f32_le(tile + ORC_TILE_ELEMS + 4 * b)", "get_f32_le(tile + ORC_TILE_ELEMS + 4 * (63 - b))")]),
    ("fp8 scales first, codes after them, pack and unpack",
     [("tile[b * ORC_BLOCK + j] = codes[j];", "tile[256 + b * ORC_BLOCK + j] = codes[j];"),
      ("put_f32_le(tile + ORC_TILE_ELEMS + 4 * b, s);", "put_f32_le(tile + 4 * b, s);"),
      ("case ORC_FP8:  return tile[i];", "case ORC_FP8:  return tile[256 + i];"),
      ("orc_dequant_fp8(tile[i], get_f32_le(tile + ORC_TILE_ELEMS + 4 * b));",
       "orc_dequant_fp8(tile[256 + i], get_f32_le(tile + 4 * b));")]),
    ("mxfp4 scales in reverse block order, pack and unpack",
     [("tile[ORC_TILE_ELEMS / 2 + b] = sc;", "tile[ORC_TILE_ELEMS / 2 + (63 - b)] = sc;"),
      ("tile[ORC_TILE_ELEMS / 2 + b]);", "tile[ORC_TILE_ELEMS / 2 + (63 - b)]);")]),
    ("mxfp4 scales first, codes after them, pack and unpack",
     [(_MX_PACK, _MX_PACK.replace("tile[i / 2]", "tile[64 + i / 2]")
                         .replace("tile[ORC_TILE_ELEMS / 2 + b]", "tile[b]")),
      (_NIBBLE_UNPACK,
       "case ORC_INT4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);\n"
       "    case ORC_MXFP4: return (uint8_t)((tile[64 + i / 2] >> (4 * (i % 2))) & 0xF);"),
      ("tile[ORC_TILE_ELEMS / 2 + b]);", "tile[b]);")]),
    ("int3 planes swapped, pack and unpack",
     [("uint8_t *q2w = tile;\n            uint8_t *q1w = tile + ORC_TILE_ELEMS / 4;",
       "uint8_t *q1w = tile;\n            uint8_t *q2w = tile + ORC_TILE_ELEMS / 8;"),
      (_INT3_UNPACK,
       "uint8_t lo = (uint8_t)((tile[ORC_TILE_ELEMS / 8 + i / 4] >> (2 * (i % 4))) & 3);\n"
       "        uint8_t hi = (uint8_t)((tile[i / 8] >> (i % 8)) & 1);")]),
    ("int3 q2w bit order, pack and unpack",
     [("q2w[i / 4] |= (uint8_t)((codes[j] & 3) << (2 * (i % 4)));",
       "q2w[i / 4] |= (uint8_t)((codes[j] & 3) << (6 - 2 * (i % 4)));"),
      (_INT3_UNPACK, _INT3_UNPACK.replace(">> (2 * (i % 4))", ">> (6 - 2 * (i % 4))"))]),
    ("int3 q1w bit order, pack and unpack",
     [("q1w[i / 8] |= (uint8_t)((codes[j] >> 2) << (i % 8));",
       "q1w[i / 8] |= (uint8_t)((codes[j] >> 2) << (7 - i % 8));"),
      (_INT3_UNPACK, _INT3_UNPACK.replace(">> (i % 8)", ">> (7 - i % 8)"))]),
    ("int3 scales big-endian, pack and unpack",
     [(_INT3_SCALE_PUT, _INT3_SCALE_PUT.replace(", sb);", ", %s);" % _swap16("sb"))),
      (_INT3_SCALE_GET, _swap16(_INT3_SCALE_GET[:-2]) + ");")]),
    ("bf16 words big-endian, pack and unpack",
     [("put_u16_le(tile + 2 * i, orc_f32_to_bf16_rne(x[i]));",
       "put_u16_le(tile + 2 * i, %s);" % _swap16("orc_f32_to_bf16_rne(x[i])")),
      ("v[i] = orc_bf16_to_f32(get_u16_le(tile + 2 * i));",
       "v[i] = orc_bf16_to_f32(%s);" % _swap16("get_u16_le(tile + 2 * i)"))]),
]

# Changes that cannot alter any result, kept out of GROUPS.
#
# Rounding fl32(x/s) instead of the exact quotient: for binary32 x and a normal
# binary16 s, a quotient that is not a half-integer lies at least ulp(x)/s from
# every half-integer (2x - (2k+1)s is a nonzero multiple of 2 ulp(x) or of ulp(s)),
# and ulp(x)/s exceeds half an ulp of the quotient because s < 2^(e_s+1).  So
# fl32(x/s) never lands on a half-integer it is not on, and RNE gives the same
# integer at both stages.
EQUIVALENT = [
    ('int rounding in float',
     [('double qd = nearbyint((double)x[j] / (double)s);',
       'double qd = nearbyintf(x[j] / s);')]),
]

# which pin files must catch each group
GROUPS = [
    (CORE, ("test_oracle_pins.py",)),
    (MXFP4, ("test_oracle_pins_mxfp4.py",)),
    (COLLECTIVES, ("test_oracle_pins_collectives.py",)),
    (F32, ("test_oracle_pins_f32.py",)),
    (LAYOUT, ("test_oracle_pins_layout.py", "test_oracle_pins.py")),
]
