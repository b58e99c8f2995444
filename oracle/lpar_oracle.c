/*
 * lpar_oracle.c -- plain, slow, single-threaded CPU oracle of the compressed
 * all-reduce (block-quantised INT4 / INT3 / FP8 codecs and a BF16 passthrough).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or constant generator with
 * the CUDA library; both follow the same written definitions and are compared
 * value by value.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * Every float operation below is one IEEE-754 binary32 operation rounded to
 * nearest-even (x86-64 SSE, no contraction); where exactness needs more range
 * the code says so and uses binary64.
 *
 * Sources (web pages, cited by title and section):
 *  [QR]   "QuickReduce INT3 Quantization and Benchmarking on MI355", sections
 *         Summary (tile of 1152 B for INT4, 896 B for INT3, 22% smaller),
 *         Method (block-level FP16 scale + symmetric quantisation; 3-bit values
 *         split into a low-2-bit plane "q2w" and a high-1-bit plane "q1w"),
 *         In practice (1 MB activation threshold for INT3).
 *  [RX]   "RCCLX: Innovating GPU communications on AMD platforms", sections
 *         Low-Precision Collectives (FP8 on the wire, up to 4:1 against FP32,
 *         computation stays in FP32) and Direct Data Access (DDA tree =
 *         reduce-scatter then all-gather).
 *  [FP8]  "FP8 Formats for Deep Learning", abstract (E4M3: 4 exponent bits,
 *         3 mantissa bits, no infinities, a single NaN mantissa pattern).
 *  [MX]   "Microscaling Data Formats for Deep Learning", abstract (a scale
 *         shared by a block of narrow floating-point elements); [QR] Summary
 *         ("INT4 and FP4" modes of the same all-reduce).
 *
 * Readings where the pages are silent (each one is listed with its reason in
 * the design notes): 32-element blocks in 2048-element tiles (the only split
 * consistent with the printed tile sizes and FP16 scales); codes stored as
 * offset binary q + 2^(b-1); scale s = f16_rne(fl32(absmax / qmax)),
 * saturating at 65504; q = RNE(x / s) of the exact quotient, clamped to
 * [-qmax, qmax]; tile byte order = codes (or planes) first, scales last, bits
 * little-endian; FP8 scale is a binary32 per 32 elements, s = fl32(a / 448),
 * encoded by multiplying with fl32(1 / s), flushed to zero below 2^-126;
 * requantisation with the same codec after the FP32 sum (the "transmitted
 * tile" of the all-gather); sum in ascending rank order from +0.0f.
 * MXFP4 (the FP4 codec): E2M1 elements, one E8M0 power-of-two scale per 32
 * elements, shared exponent floor(log2(absmax)) - 2 (2 = the largest E2M1
 * exponent) clamped to [-127, 127], elements RNE(x / 2^E) saturated at +-6;
 * tile = 1024 B of nibbles (element 2k low) then 64 scale bytes.
 */
#include "lpar_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Number formats.                                                           */
/* ------------------------------------------------------------------------- */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/*
 * Round a >= 0 (finite) to the nearest value of a binary floating-point format
 * whose significand has p bits (hidden bit included) and whose smallest normal
 * exponent is emin, ties to even.  Values below 2^emin land on the subnormal
 * grid 2^(emin-p+1).  No overflow handling: the caller compares the result with
 * the format's largest finite value.  Exact: a / quantum only moves the binary
 * point, and nearbyint() rounds a binary64 to an integer ties-to-even.
 */
static double round_to_format(double a, int p, int emin)
{
    if (a == 0.0) return 0.0;
    int E;
    frexp(a, &E);                 /* a = m * 2^E, m in [0.5, 1): leading bit is 2^(E-1) */
    int e = E - 1;
    if (e < emin) e = emin;       /* subnormal range shares the grid of 2^emin */
    double quantum = ldexp(1.0, e - (p - 1));
    return nearbyint(a / quantum) * quantum;
}

/* Encode a value already on the grid of a (p, emin, bias) format into bits. */
static uint32_t encode_on_grid(double r, int p, int emin, int bias)
{
    if (r == 0.0) return 0;
    int E;
    frexp(r, &E);
    int e = E - 1;
    if (e < emin) {               /* subnormal: exponent field 0 */
        return (uint32_t)(r / ldexp(1.0, emin - (p - 1)));
    }
    uint32_t mant = (uint32_t)(r / ldexp(1.0, e - (p - 1))) - (1u << (p - 1));
    return ((uint32_t)(e + bias) << (p - 1)) | mant;
}

float orc_bf16_to_f32(uint16_t h)
{
    /* bfloat16 is the upper half of a binary32. */
    return bits_to_f32((uint32_t)h << 16);
}

uint16_t orc_f32_to_bf16_rne(float x)
{
    uint32_t u = f32_to_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
    /* bfloat16: 8 significand bits, emin -126, bias 127, largest finite (2-2^-7)*2^127. */
    double r = round_to_format(fabs((double)x), 8, -126);
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127)) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | encode_on_grid(r, 8, -126, 127));
}

uint16_t orc_f32_to_f16_rne(float x)
{
    uint32_t u = f32_to_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(x)) return (uint16_t)(sign | 0x7C00u);
    /* binary16: 11 significand bits, emin -14, bias 15, largest finite 65504. */
    double r = round_to_format(fabs((double)x), 11, -14);
    if (r > 65504.0) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | encode_on_grid(r, 11, -14, 15));
}

float orc_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ef = (h >> 10) & 0x1F;
    int mf = h & 0x3FF;
    double v;
    if (ef == 0x1F) {
        v = mf ? NAN : INFINITY;
    } else if (ef == 0) {
        v = ldexp((double)mf, -24);                     /* 0.m * 2^-14 */
    } else {
        v = ldexp(1.0 + (double)mf / 1024.0, ef - 15);
    }
    return (float)(sign ? -v : v);
}

/*
 * E4M3 per [FP8]: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * S.1111.111 is the only NaN pattern, so S.1111.110 = 1.75 * 2^8 = 448 is the
 * largest finite magnitude; exponent field 0 holds subnormals 0.mmm * 2^-6.
 */
float orc_e4m3_to_f32(uint8_t e)
{
    int sign = (e >> 7) & 1;
    int ef = (e >> 3) & 0xF;
    int mf = e & 0x7;
    double v;
    if (ef == 0xF && mf == 0x7) return NAN;
    if (ef == 0) v = ldexp((double)mf / 8.0, -6);
    else         v = ldexp(1.0 + (double)mf / 8.0, ef - 7);
    return (float)(sign ? -v : v);
}

/* f32 -> E4M3, round to nearest even, finite results saturate at +-448. */
uint8_t orc_f32_to_e4m3_rne_satfinite(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = (f32_to_bits(x) >> 31) ? 0x80 : 0x00;
    double a = fabs((double)x);
    double r = isinf(x) ? 448.0 : round_to_format(a, 4, -6);
    if (r > 448.0) r = 448.0;
    return (uint8_t)(sign | encode_on_grid(r, 4, -6, 7));
}

/*
 * E2M1 (the MX FP4 element): 1 sign, 2 exponent (bias 1), 1 mantissa bit; no
 * infinities or NaN.  Exponent field 0 holds the subnormal 0.m * 2^0, so the
 * magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4 and 6.
 */
float orc_e2m1_to_f32(uint8_t c)
{
    int sign = (c >> 3) & 1;
    int ef = (c >> 1) & 3;
    int mf = c & 1;
    double v = (ef == 0) ? 0.5 * mf : ldexp(1.0 + 0.5 * mf, ef - 1);
    return (float)(sign ? -v : v);
}

/* A real value (binary64, exact) -> E2M1, round to nearest even, magnitudes
 * above 6 saturate to 6; the sign is kept (a negative value that rounds to
 * zero gives the negative-zero code 0x8). */
uint8_t orc_e2m1_rne_satfinite(double y)
{
    uint8_t sign = signbit(y) ? 0x8 : 0x0;
    double r = round_to_format(fabs(y), 2, 0);
    if (r > 6.0) r = 6.0;
    return (uint8_t)(sign | encode_on_grid(r, 2, 0, 1));
}

/* E8M0 scale code -> 2^(code - 127) (code 255, the NaN pattern, is never produced). */
double orc_e8m0_to_f64(uint8_t code) { return ldexp(1.0, (int)code - 127); }

/* ------------------------------------------------------------------------- */
/* Tile geometry ([QR] Summary: 1152 B INT4, 896 B INT3 per transmitted tile). */
/* ------------------------------------------------------------------------- */

size_t orc_tile_bytes(int codec)
{
    switch (codec) {
    case ORC_BF16: return ORC_TILE_ELEMS * 2;                        /* 4096 */
    case ORC_FP8:  return ORC_TILE_ELEMS + ORC_BLOCKS_PER_TILE * 4;  /* 2048 + 256 = 2304 */
    case ORC_INT4: return ORC_TILE_ELEMS / 2 + ORC_BLOCKS_PER_TILE * 2;       /* 1024 + 128 = 1152 */
    case ORC_INT3: return ORC_TILE_ELEMS / 4 + ORC_TILE_ELEMS / 8
                        + ORC_BLOCKS_PER_TILE * 2;                   /* 512 + 256 + 128 = 896 */
    case ORC_MXFP4: return ORC_TILE_ELEMS / 2 + ORC_BLOCKS_PER_TILE;  /* 1024 + 64 = 1088 */
    default: return 0;
    }
}

size_t orc_wire_bytes(int codec, size_t n) { return (n / ORC_TILE_ELEMS) * orc_tile_bytes(codec); }

/* ------------------------------------------------------------------------- */
/* Block quantiser ([QR] Method: block-level FP16 scale, symmetric codes).    */
/* ------------------------------------------------------------------------- */

void orc_quant_block_int(const float *x, int bits, uint16_t *scale_bits, uint8_t *codes)
{
    const int qmax = (1 << (bits - 1)) - 1;      /* 7 for INT4, 3 for INT3 */
    const int bias = 1 << (bits - 1);            /* offset-binary code = q + bias */

    float a = 0.0f;                              /* 1. block absmax */
    for (int j = 0; j < ORC_BLOCK; ++j) {
        float m = fabsf(x[j]);
        if (m > a) a = m;
    }
    float ratio = a / (float)qmax;               /* 2. one binary32 division ... */
    uint16_t sb = orc_f32_to_f16_rne(ratio);     /*    ... then binary16 RNE */
    if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFF;  /*    saturate at 65504 */
    float s = orc_f16_to_f32(sb);

    for (int j = 0; j < ORC_BLOCK; ++j) {        /* 3. q = clamp(RNE(x / s)) */
        int q = 0;
        if (s != 0.0f) {
            /* binary64 holds x/s within 2^-50 relative, far closer than any
             * non-tie quotient of a 24-bit x by an 11-bit s comes to a tie. */
            double qd = nearbyint((double)x[j] / (double)s);
            if (qd > qmax) qd = qmax;
            if (qd < -qmax) qd = -qmax;
            q = (int)qd;
        }
        codes[j] = (uint8_t)(q + bias);          /* 4. offset binary */
    }
    *scale_bits = sb;
}

float orc_dequant_int(uint8_t code, int bits, uint16_t scale_bits)
{
    int q = (int)code - (1 << (bits - 1));
    return (float)q * orc_f16_to_f32(scale_bits);   /* exact: <= 4-bit x 11-bit */
}

void orc_quant_block_fp8(const float *x, float *scale, uint8_t *codes)
{
    float a = 0.0f;
    for (int j = 0; j < ORC_BLOCK; ++j) {
        float m = fabsf(x[j]);
        if (m > a) a = m;
    }
    float s = a / 448.0f;                        /* largest finite E4M3 */
    if (s < 0x1p-126f) {                         /* zero or subnormal scale: zero block */
        for (int j = 0; j < ORC_BLOCK; ++j) codes[j] = 0x00;
        *scale = 0.0f;
        return;
    }
    float inv = 1.0f / s;
    for (int j = 0; j < ORC_BLOCK; ++j) {
        float y = x[j] * inv;
        codes[j] = orc_f32_to_e4m3_rne_satfinite(y);
    }
    *scale = s;
}

float orc_dequant_fp8(uint8_t code, float scale)
{
    return orc_e4m3_to_f32(code) * scale;        /* one binary32 multiply */
}

/*
 * MXFP4 block ([MX]): the shared exponent E is the largest power of two that
 * the block's absmax reaches, minus the largest E2M1 exponent (2), so the
 * absmax lands in [4, 8) after scaling; E is clamped to the E8M0 range
 * [-127, 127] (an all-zero block takes the bottom of the range).  Each element
 * is x / 2^E (exact in binary64) rounded to E2M1.
 */
void orc_quant_block_mxfp4(const float *x, uint8_t *scale_code, uint8_t *codes)
{
    float a = 0.0f;
    for (int j = 0; j < ORC_BLOCK; ++j) {
        float m = fabsf(x[j]);
        if (m > a) a = m;
    }
    int E = -127;
    if (a > 0.0f) {
        int F;
        frexp((double)a, &F);                    /* a = m * 2^F, m in [0.5, 1): floor(log2 a) = F - 1 */
        E = (F - 1) - 2;
        if (E < -127) E = -127;
        if (E > 127) E = 127;
    }
    for (int j = 0; j < ORC_BLOCK; ++j) codes[j] = orc_e2m1_rne_satfinite(ldexp((double)x[j], -E));
    *scale_code = (uint8_t)(E + 127);
}

float orc_dequant_mxfp4(uint8_t code, uint8_t scale_code)
{
    /* exact: a 2-bit significand times a power of two in [2^-127, 2^125] */
    return (float)((double)orc_e2m1_to_f32(code) * orc_e8m0_to_f64(scale_code));
}

/* ------------------------------------------------------------------------- */
/* Tile packing (byte layout is a reading: codes/planes first, scales last).  */
/* ------------------------------------------------------------------------- */

static void put_u16_le(uint8_t *p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static uint16_t get_u16_le(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void put_f32_le(uint8_t *p, float f)
{
    uint32_t u = f32_to_bits(f);
    p[0] = (uint8_t)u; p[1] = (uint8_t)(u >> 8); p[2] = (uint8_t)(u >> 16); p[3] = (uint8_t)(u >> 24);
}
static float get_f32_le(const uint8_t *p)
{
    return bits_to_f32((uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24));
}

/* Quantise one 2048-element tile of binary32 values into tile bytes. */
void orc_quant_tile(const float *x, int codec, uint8_t *tile)
{
    memset(tile, 0, orc_tile_bytes(codec));
    if (codec == ORC_BF16) {
        for (int i = 0; i < ORC_TILE_ELEMS; ++i) put_u16_le(tile + 2 * i, orc_f32_to_bf16_rne(x[i]));
        return;
    }
    for (int b = 0; b < ORC_BLOCKS_PER_TILE; ++b) {
        uint8_t codes[ORC_BLOCK];
        const float *xb = x + b * ORC_BLOCK;
        if (codec == ORC_FP8) {
            float s;
            orc_quant_block_fp8(xb, &s, codes);
            for (int j = 0; j < ORC_BLOCK; ++j) tile[b * ORC_BLOCK + j] = codes[j];
            put_f32_le(tile + ORC_TILE_ELEMS + 4 * b, s);
        } else if (codec == ORC_MXFP4) {
            uint8_t sc;
            orc_quant_block_mxfp4(xb, &sc, codes);
            for (int j = 0; j < ORC_BLOCK; ++j) {
                int i = b * ORC_BLOCK + j;
                tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));
            }
            tile[ORC_TILE_ELEMS / 2 + b] = sc;
        } else if (codec == ORC_INT4) {
            uint16_t sb;
            orc_quant_block_int(xb, 4, &sb, codes);
            for (int j = 0; j < ORC_BLOCK; ++j) {
                int i = b * ORC_BLOCK + j;               /* element index in tile */
                tile[i / 2] |= (uint8_t)(codes[j] << (4 * (i % 2)));
            }
            put_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b, sb);
        } else { /* ORC_INT3: q2w plane = code & 3, q1w plane = code >> 2 */
            uint16_t sb;
            orc_quant_block_int(xb, 3, &sb, codes);
            uint8_t *q2w = tile;
            uint8_t *q1w = tile + ORC_TILE_ELEMS / 4;
            for (int j = 0; j < ORC_BLOCK; ++j) {
                int i = b * ORC_BLOCK + j;
                q2w[i / 4] |= (uint8_t)((codes[j] & 3) << (2 * (i % 4)));
                q1w[i / 8] |= (uint8_t)((codes[j] >> 2) << (i % 8));
            }
            put_u16_le(tile + ORC_TILE_ELEMS / 4 + ORC_TILE_ELEMS / 8 + 2 * b, sb);
        }
    }
}

/* Read element i's code back out of a tile (inverse of the packing above). */
uint8_t orc_tile_code(const uint8_t *tile, int codec, int i)
{
    switch (codec) {
    case ORC_FP8:  return tile[i];
    case ORC_INT4:
    case ORC_MXFP4: return (uint8_t)((tile[i / 2] >> (4 * (i % 2))) & 0xF);
    case ORC_INT3: {
        uint8_t lo = (uint8_t)((tile[i / 4] >> (2 * (i % 4))) & 3);
        uint8_t hi = (uint8_t)((tile[ORC_TILE_ELEMS / 4 + i / 8] >> (i % 8)) & 1);
        return (uint8_t)(lo | (hi << 2));
    }
    default: return 0;
    }
}

/* Dequantise one tile into binary32 values. */
void orc_dequant_tile(const uint8_t *tile, int codec, float *v)
{
    for (int i = 0; i < ORC_TILE_ELEMS; ++i) {
        int b = i / ORC_BLOCK;
        switch (codec) {
        case ORC_BF16:
            v[i] = orc_bf16_to_f32(get_u16_le(tile + 2 * i));
            break;
        case ORC_FP8:
            v[i] = orc_dequant_fp8(tile[i], get_f32_le(tile + ORC_TILE_ELEMS + 4 * b));
            break;
        case ORC_INT4:
            v[i] = orc_dequant_int(orc_tile_code(tile, codec, i), 4,
                                   get_u16_le(tile + ORC_TILE_ELEMS / 2 + 2 * b));
            break;
        case ORC_INT3:
            v[i] = orc_dequant_int(orc_tile_code(tile, codec, i), 3,
                                   get_u16_le(tile + ORC_TILE_ELEMS / 4 + ORC_TILE_ELEMS / 8 + 2 * b));
            break;
        case ORC_MXFP4:
            v[i] = orc_dequant_mxfp4(orc_tile_code(tile, codec, i), tile[ORC_TILE_ELEMS / 2 + b]);
            break;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* The three stages and the two-shot all-reduce ([RX] DDA tree: reduce-       */
/* scatter then all-gather; [RX] Low-Precision: the sum is taken in FP32).    */
/* ------------------------------------------------------------------------- */

/* Stage 1: every tile of one rank's BF16 message into its wire. */
void orc_quantize(const uint16_t *in_bf16, size_t n, int codec, uint8_t *wire)
{
    float x[ORC_TILE_ELEMS];
    size_t tb = orc_tile_bytes(codec);
    for (size_t t = 0; t < n / ORC_TILE_ELEMS; ++t) {
        for (int i = 0; i < ORC_TILE_ELEMS; ++i) x[i] = orc_bf16_to_f32(in_bf16[t * ORC_TILE_ELEMS + i]);
        orc_quant_tile(x, codec, wire + t * tb);
    }
}

/*
 * Stage 2 (the reducer of one shard): for every tile index t in
 * [tile_begin, tile_begin + tile_count), dequantise tile t of each of the N
 * wires, sum in binary32 in ascending rank order starting from +0.0f, and
 * requantise the sums with the same codec into tile t of wire_out.
 */
void orc_reduce(const uint8_t *const *wires, int N, size_t tile_begin, size_t tile_count,
                int codec, uint8_t *wire_out)
{
    float acc[ORC_TILE_ELEMS], v[ORC_TILE_ELEMS];
    size_t tb = orc_tile_bytes(codec);
    for (size_t t = tile_begin; t < tile_begin + tile_count; ++t) {
        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = +0.0f;
        for (int r = 0; r < N; ++r) {
            orc_dequant_tile(wires[r] + t * tb, codec, v);
            for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];
        }
        orc_quant_tile(acc, codec, wire_out + t * tb);
    }
}

/* Stage 3 (all-gather receiver): wire -> BF16, round to nearest even. */
void orc_decode(const uint8_t *wire, size_t n, int codec, uint16_t *out_bf16)
{
    float v[ORC_TILE_ELEMS];
    size_t tb = orc_tile_bytes(codec);
    for (size_t t = 0; t < n / ORC_TILE_ELEMS; ++t) {
        orc_dequant_tile(wire + t * tb, codec, v);
        for (int i = 0; i < ORC_TILE_ELEMS; ++i) out_bf16[t * ORC_TILE_ELEMS + i] = orc_f32_to_bf16_rne(v[i]);
    }
}

/*
 * Whole collective.  The per-rank message is 2n bytes of BF16; a quantising
 * codec runs only when 2n >= min_quant_bytes ([QR] In practice: 1 MB
 * activation threshold), otherwise the BF16 passthrough runs.  Returns the
 * codec actually used, or -1 on a bad argument or allocation failure.
 */
int orc_allreduce(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                  uint16_t *const *out_bf16, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || n % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    if (codec != ORC_BF16 && 2 * n < min_quant_bytes) codec = ORC_BF16;
    size_t wb = orc_wire_bytes(codec, n);
    size_t tiles = n / ORC_TILE_ELEMS;
    uint8_t *wires[ORC_MAX_RANKS];
    uint8_t *gather = (uint8_t *)malloc(wb ? wb : 1);
    if (!gather) return -1;
    for (int r = 0; r < N; ++r) {
        wires[r] = (uint8_t *)malloc(wb ? wb : 1);
        if (!wires[r]) { for (int k = 0; k < r; ++k) free(wires[k]); free(gather); return -1; }
        if (codec == ORC_BF16) memcpy(wires[r], in_bf16[r], wb);     /* the wire is the input */
        else orc_quantize(in_bf16[r], n, codec, wires[r]);            /* stage 1 */
    }
    /* Reduce-scatter: shard j owns tiles [jT/N, (j+1)T/N); each shard's reducer
     * reads its tile indices from all N wires. */
    for (int j = 0; j < N; ++j) {
        size_t t0 = (size_t)j * tiles / (size_t)N, t1 = (size_t)(j + 1) * tiles / (size_t)N;
        orc_reduce((const uint8_t *const *)wires, N, t0, t1 - t0, codec, gather);
    }
    /* All-gather: every rank decodes the whole gathered wire. */
    for (int r = 0; r < N; ++r) orc_decode(gather, n, codec, out_bf16[r]);
    for (int r = 0; r < N; ++r) free(wires[r]);
    free(gather);
    return codec;
}

/* ------------------------------------------------------------------------- */
/* Standalone low-precision collectives ([RX] Low-Precision Collectives: the   */
/* quantised wire is used by the other collectives too) and the one-shot       */
/* all-reduce ([RX] Direct Data Access, "flat": every rank reduces all inputs  */
/* itself).  Each rank's message is quantised once (stage 1); the receiver     */
/* dequantises.  A reduction sums in binary32 in ascending rank order from     */
/* +0.0f and rounds the sum once to BF16 (no second quantisation: nothing is   */
/* transmitted after it).                                                       */
/* ------------------------------------------------------------------------- */

/* Quantise every rank's message (or copy it for BF16) into freshly allocated
 * wires; returns 0 on success. */
static int quantize_all(const uint16_t *const *in_bf16, int N, size_t n, int codec, uint8_t **wires)
{
    size_t wb = orc_wire_bytes(codec, n);
    for (int r = 0; r < N; ++r) {
        wires[r] = (uint8_t *)malloc(wb ? wb : 1);
        if (!wires[r]) { for (int k = 0; k < r; ++k) free(wires[k]); return -1; }
        if (codec == ORC_BF16) memcpy(wires[r], in_bf16[r], wb);
        else orc_quantize(in_bf16[r], n, codec, wires[r]);
    }
    return 0;
}

/* BF16 sum of tile t over the N wires (acc from +0.0f, ranks ascending). */
static void reduce_tile_to_bf16(uint8_t *const *wires, int N, size_t t, int codec, uint16_t *dst)
{
    float acc[ORC_TILE_ELEMS], v[ORC_TILE_ELEMS];
    size_t tb = orc_tile_bytes(codec);
    for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = +0.0f;
    for (int r = 0; r < N; ++r) {
        orc_dequant_tile(wires[r] + t * tb, codec, v);
        for (int i = 0; i < ORC_TILE_ELEMS; ++i) acc[i] = acc[i] + v[i];
    }
    for (int i = 0; i < ORC_TILE_ELEMS; ++i) dst[i] = orc_f32_to_bf16_rne(acc[i]);
}

static int effective(int codec, size_t message_bytes, size_t min_quant_bytes)
{
    return (codec != ORC_BF16 && message_bytes < min_quant_bytes) ? ORC_BF16 : codec;
}

/*
 * Reduce-scatter: rank j receives tiles [jT/N, (j+1)T/N) of the sum (the same
 * floor partition as the all-reduce's shards), as BF16, in out_bf16[j] from
 * element 0.  Threshold on the per-rank message 2n.
 */
int orc_reduce_scatter(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                       uint16_t *const *out_bf16, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || n % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    codec = effective(codec, 2 * n, min_quant_bytes);
    uint8_t *wires[ORC_MAX_RANKS];
    if (quantize_all(in_bf16, N, n, codec, wires)) return -1;
    size_t T = n / ORC_TILE_ELEMS;
    for (int j = 0; j < N; ++j) {
        size_t t0 = (size_t)j * T / (size_t)N, t1 = (size_t)(j + 1) * T / (size_t)N;
        for (size_t t = t0; t < t1; ++t)
            reduce_tile_to_bf16(wires, N, t, codec, out_bf16[j] + (t - t0) * ORC_TILE_ELEMS);
    }
    for (int r = 0; r < N; ++r) free(wires[r]);
    return codec;
}

/* One-shot all-reduce: every rank receives the whole BF16 sum. */
int orc_allreduce_oneshot(const uint16_t *const *in_bf16, int N, size_t n, int codec,
                          uint16_t *const *out_bf16, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || n % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    codec = effective(codec, 2 * n, min_quant_bytes);
    uint8_t *wires[ORC_MAX_RANKS];
    if (quantize_all(in_bf16, N, n, codec, wires)) return -1;
    for (size_t t = 0; t < n / ORC_TILE_ELEMS; ++t)
        for (int r = 0; r < N; ++r)
            reduce_tile_to_bf16(wires, N, t, codec, out_bf16[r] + t * ORC_TILE_ELEMS);
    for (int r = 0; r < N; ++r) free(wires[r]);
    return codec;
}

/*
 * All-gather: rank r contributes m elements; every rank j receives all N
 * contributions, rank r's at elements [r*m, (r+1)*m) of out_bf16[j], each the
 * BF16 decode of rank r's wire.  Threshold on the per-rank message 2m.
 */
int orc_all_gather(const uint16_t *const *in_bf16, int N, size_t m, int codec,
                   uint16_t *const *out_bf16, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || m % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    codec = effective(codec, 2 * m, min_quant_bytes);
    uint8_t *wires[ORC_MAX_RANKS];
    if (quantize_all(in_bf16, N, m, codec, wires)) return -1;
    for (int r = 0; r < N; ++r)
        for (int j = 0; j < N; ++j) {
            if (codec == ORC_BF16) memcpy(out_bf16[j] + (size_t)r * m, wires[r], 2 * m);
            else orc_decode(wires[r], m, codec, out_bf16[j] + (size_t)r * m);
        }
    for (int r = 0; r < N; ++r) free(wires[r]);
    return codec;
}

/*
 * All-to-all: rank r's message is N segments of m elements, segment j bound
 * for rank j; rank j receives rank r's segment j at elements [r*m, (r+1)*m)
 * of out_bf16[j], the BF16 decode of that part of rank r's wire.  Threshold
 * on the per-rank message 2*N*m.
 */
int orc_all_to_all(const uint16_t *const *in_bf16, int N, size_t m, int codec,
                   uint16_t *const *out_bf16, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || m % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    size_t n = (size_t)N * m;
    codec = effective(codec, 2 * n, min_quant_bytes);
    uint8_t *wires[ORC_MAX_RANKS];
    if (quantize_all(in_bf16, N, n, codec, wires)) return -1;
    size_t seg_wire = orc_wire_bytes(codec, m);
    for (int r = 0; r < N; ++r)
        for (int j = 0; j < N; ++j) {
            const uint8_t *seg = wires[r] + (size_t)j * seg_wire;
            if (codec == ORC_BF16) memcpy(out_bf16[j] + (size_t)r * m, seg, 2 * m);
            else orc_decode(seg, m, codec, out_bf16[j] + (size_t)r * m);
        }
    for (int r = 0; r < N; ++r) free(wires[r]);
    return codec;
}

/* ------------------------------------------------------------------------- */
/* FP32 messages ([RX] Low-Precision Collectives: FP32 or BF16 inputs, FP8 on  */
/* the wire, "up to 4:1" against FP32).  The same tiles and stages; the input  */
/* blocks are binary32 values, and the result is the dequantised gathered     */
/* value itself (binary32, no rounding).  The uncompressed passthrough sums   */
/* the binary32 inputs in rank order from +0.0f.                               */
/* ------------------------------------------------------------------------- */
int orc_allreduce_f32(const float *const *in_f32, int N, size_t n, int codec,
                      float *const *out_f32, size_t min_quant_bytes)
{
    if (N < 1 || N > ORC_MAX_RANKS || n % ORC_TILE_ELEMS != 0) return -1;
    if (codec < ORC_BF16 || codec > ORC_MXFP4) return -1;
    codec = effective(codec, 4 * n, min_quant_bytes);
    size_t tiles = n / ORC_TILE_ELEMS;
    if (codec == ORC_BF16) {                     /* passthrough: exact binary32 sum */
        for (size_t i = 0; i < n; ++i) {
            float acc = +0.0f;
            for (int r = 0; r < N; ++r) acc = acc + in_f32[r][i];
            for (int r = 0; r < N; ++r) out_f32[r][i] = acc;
        }
        return codec;
    }
    size_t tb = orc_tile_bytes(codec), wb = tiles * tb;
    uint8_t *wires[ORC_MAX_RANKS];
    uint8_t *gather = (uint8_t *)malloc(wb ? wb : 1);
    if (!gather) return -1;
    for (int r = 0; r < N; ++r) {
        wires[r] = (uint8_t *)malloc(wb ? wb : 1);
        if (!wires[r]) { for (int k = 0; k < r; ++k) free(wires[k]); free(gather); return -1; }
        for (size_t t = 0; t < tiles; ++t)
            orc_quant_tile(in_f32[r] + t * ORC_TILE_ELEMS, codec, wires[r] + t * tb);     /* stage 1 */
    }
    for (int j = 0; j < N; ++j) {                /* reduce-scatter shards, as in orc_allreduce */
        size_t t0 = (size_t)j * tiles / (size_t)N, t1 = (size_t)(j + 1) * tiles / (size_t)N;
        orc_reduce((const uint8_t *const *)wires, N, t0, t1 - t0, codec, gather);
    }
    for (size_t t = 0; t < tiles; ++t)            /* all-gather: the dequantised values */
        for (int r = 0; r < N; ++r) orc_dequant_tile(gather + t * tb, codec, out_f32[r] + t * ORC_TILE_ELEMS);
    for (int r = 0; r < N; ++r) free(wires[r]);
    free(gather);
    return codec;
}
