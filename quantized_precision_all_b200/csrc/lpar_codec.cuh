// lpar_codec.cuh -- per-block codec arithmetic for sm_100a (device code only).
//
// One thread owns one 32-element block: absmax, scale, codes and packing stay
// in registers, so no warp shuffles are needed and the per-block division is
// paid once per 32 elements.
//
// Formats ("QuickReduce INT3 Quantization and Benchmarking on MI355", Summary
// and Method; "RCCLX: Innovating GPU communications on AMD platforms",
// Low-Precision Collectives; "FP8 Formats for Deep Learning", abstract):
//   INT4/INT3: s = f16_rne(fl32(absmax / qmax)) saturating at 65504,
//              q = clamp(RNE(x / s)) of the exact quotient, code = q + 2^(b-1).
//   FP8 E4M3:  s = fl32(absmax / 448), zero block when s < 2^-126,
//              code = e4m3_rne_satfinite(fl32(x * fl32(1 / s))).
//
// Exact RNE(x / s) without a per-element division.  With h = fl(x * fl(1/s))
// (relative error < 2^-22) let k = RNE(h - 1/2); k is RNE(x/s) or one less.
// m = (k + 1/2) * s is exact in binary32 ((2k+1) has <= 5 bits, s <= 11 bits),
// so comparing x with m decides the last step exactly: q = k + 1 when x > m,
// or when x == m (a tie) and k is odd (ties to even); otherwise q = k.
// k is found with the add-magic trick: fl(h' + (1.5*2^23 + bias)) puts
// k + bias in the low mantissa bits, which is the offset-binary code itself.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace lpar {

constexpr int kBlock = 32;
constexpr int kTileElems = 2048;
constexpr int kBlocksPerTile = 64;

enum CodecId : int { kBF16 = 0, kFP8 = 1, kINT4 = 2, kINT3 = 3 };

// Byte layout of one 2048-element tile.
template <int C> struct Layout;
template <> struct Layout<kINT4> {
    static constexpr int kTileBytes = 1152, kScaleOff = 1024, kBits = 4;
};
template <> struct Layout<kINT3> {
    static constexpr int kTileBytes = 896, kQ1wOff = 512, kScaleOff = 768, kBits = 3;
};
template <> struct Layout<kFP8> {
    static constexpr int kTileBytes = 2304, kScaleOff = 2048;
};
template <> struct Layout<kBF16> {
    static constexpr int kTileBytes = 4096;
};

// The packed payload of one block (codes + scale) as it sits in a tile.
template <int C> struct Packed;
template <> struct Packed<kINT4> { uint32_t w[4]; uint16_t scale; };          // 16 B codes
template <> struct Packed<kINT3> { uint32_t q2w[2]; uint32_t q1w; uint16_t scale; };
template <> struct Packed<kFP8> { uint32_t w[8]; float scale; };              // 32 B codes

// ---------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two binary32 -> packed BF16x2, round to nearest even; lo lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two binary32 -> packed E4M3x2, RNE, finite saturation; lo lands in bits 0..7.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// Packed E4M3x2 (16 bits) -> two exact binary32 values (E4M3 is a subset of binary16).
__device__ __forceinline__ void unpack_e4m3x2(uint32_t two, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)two));
    lo = __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFF)));
    hi = __half2float(__ushort_as_half((uint16_t)(h2 >> 16)));
}

// Maximum of |bf16| over a packed pair, as a packed pair; the sign bits are
// junk and are masked off by the caller.
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// absmax of 32 BF16 values held as 16 packed words -> binary32 (exact).
__device__ __forceinline__ float absmax_bf16x32(const uint32_t (&w)[16]) {
    uint32_t m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = maxabs_bf16x2(w[2 * i], w[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = maxabs_bf16x2(m[2 * i], m[2 * i + 1]);
    m[0] = maxabs_bf16x2(m[0], m[1]);
    m[2] = maxabs_bf16x2(m[2], m[3]);
    m[0] = maxabs_bf16x2(m[0], m[2]);
    uint32_t lo = m[0] & 0x7FFFu, hi = (m[0] >> 16) & 0x7FFFu;
    return __uint_as_float((lo > hi ? lo : hi) << 16);
}

__device__ __forceinline__ float absmax_f32x32(const float (&x)[32]) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        a0 = fmaxf(a0, fabsf(x[j]));
        a1 = fmaxf(a1, fabsf(x[j + 1]));
        a2 = fmaxf(a2, fabsf(x[j + 2]));
        a3 = fmaxf(a3, fabsf(x[j + 3]));
    }
    return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// ---------------------------------------------------------------------------
// INT4 / INT3 block quantiser.  x[32] in binary32 (exact BF16 values at stage 1,
// FP32 sums at stage 2), a = max|x|.
// ---------------------------------------------------------------------------
struct IntScale {
    uint16_t bits;   // binary16 scale as stored in the tile
    float s;         // its value
    float r;         // fl(1/s), or 0 when s == 0
    float hs;        // s/2, or +inf when s == 0 (nothing ever rounds up)
    float lim;       // (qmax + 1) * s: bound applied on the slow path
    bool fast;       // normal, unsaturated scale: |x/s| <= qmax (1 + 2^-11), no clamp needed
};

template <int BITS>
__device__ __forceinline__ IntScale int_scale(float a) {
    constexpr int kQmax = (1 << (BITS - 1)) - 1;
    IntScale k;
    const float ratio = __fdiv_rn(a, (float)kQmax);                  // one IEEE division per block
    uint16_t sb = __half_as_ushort(__float2half_rn(ratio));
    if (sb == 0x7C00u) sb = 0x7BFFu;                                   // saturate at 65504
    k.bits = sb;
    k.s = __half2float(__ushort_as_half(sb));
    k.fast = (sb >= 0x0400u) && (sb != 0x7BFFu);
    k.r = (k.s != 0.f) ? __frcp_rn(k.s) : 0.f;
    k.hs = (k.s != 0.f) ? 0.5f * k.s : __int_as_float(0x7F800000);
    k.lim = (float)(kQmax + 1) * k.s;                                 // exact
    return k;
}

// Offset-binary code of one element (low byte) and, when wanted, q * s.
template <int BITS, bool FAST, bool WANT_V>
__device__ __forceinline__ uint32_t int_code(float x, const IntScale &k, float &v) {
    constexpr int kQmax = (1 << (BITS - 1)) - 1;
    constexpr int kBias = 1 << (BITS - 1);
    const float magic = 12582912.0f + (float)kBias;                   // 1.5 * 2^23 + bias
    if (!FAST) x = fminf(fmaxf(x, -k.lim), k.lim);                    // keeps |x/s| <= qmax + 1
    const float hm = __fmaf_rn(x, k.r, -0.5f);                        // ~ x/s - 1/2
    const float C = __fadd_rn(hm, magic);                             // magic + RNE(hm)
    const float kf = __fsub_rn(C, magic);                             // k, exactly
    const float m = __fmaf_rn(kf, k.s, k.hs);                         // (k + 1/2) s, exact
    uint32_t c = __float_as_uint(C) - 0x4B400000u;                    // k + bias
    const bool up = (x > m) || ((x == m) && (c & 1u));               // bias is even: parity of k
    c += up ? 1u : 0u;
    if (!FAST) c = (uint32_t)min(max((int)c, kBias - kQmax), kBias + kQmax);
    if (WANT_V) {
        if (FAST) v = __fmaf_rn(kf, k.s, up ? k.s : 0.f);             // (k + up) s, exact
        else v = __fmul_rn((float)((int)c - kBias), k.s);
    }
    return c;
}

// INT4: 8 codes of elements 8i..8i+7 -> one word (element 8i in the low nibble).
template <bool FAST, bool WANT_V>
__device__ __forceinline__ void int4_body(const float (&x)[32], const IntScale &k, uint32_t (&w)[4],
                                          uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t c[8];
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = int_code<4, FAST, WANT_V>(x[8 * i + j], k, v[j]);
        const uint32_t b0 = c[0] | (c[1] << 4), b1 = c[2] | (c[3] << 4);
        const uint32_t b2 = c[4] | (c[5] << 4), b3 = c[6] | (c[7] << 4);
        w[i] = __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
        if (WANT_V) {
#pragma unroll
            for (int q = 0; q < 4; ++q) o[4 * i + q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
        }
    }
}

// INT3: 4 codes of elements 4g..4g+3 -> q2w byte g (2 bits each) and q1w bits 4g..4g+3.
template <bool FAST, bool WANT_V>
__device__ __forceinline__ void int3_body(const float (&x)[32], const IntScale &k, uint32_t (&q2w)[2],
                                          uint32_t &q1w, uint32_t (&o)[16]) {
    q2w[0] = q2w[1] = 0u;
    q1w = 0u;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        uint32_t c[4];
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) c[j] = int_code<3, FAST, WANT_V>(x[4 * g + j], k, v[j]);
        const uint32_t w = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
        uint32_t lo = w & 0x03030303u;                 // low two bits of each code, one per byte
        lo |= lo >> 6;                                 // element 4g+1 -> bits 2..3
        lo |= lo >> 12;                                // elements 4g+2, 4g+3 -> bits 4..7
        q2w[g >> 2] |= (lo & 0xFFu) << (8 * (g & 3));
        const uint32_t hb = (w >> 2) & 0x01010101u;    // high bit of each code, one per byte
        q1w |= ((hb * 0x01020408u) >> 24) << (4 * g);  // gather the 4 bits (no carries)
        if (WANT_V) {
            o[2 * g] = pack_bf16x2(v[0], v[1]);
            o[2 * g + 1] = pack_bf16x2(v[2], v[3]);
        }
    }
}

// ---------------------------------------------------------------------------
// Dequantise one block and add it to acc[32] (acc = fl32(acc + q*s); the
// product is exact for INT codes, so one FMA rounds exactly once).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float magic_code_to_float(uint32_t bytes, int b) {
    // byte b of `bytes` as the low mantissa bits of 2^23: value 2^23 + byte
    return __uint_as_float(__byte_perm(bytes, 0x4B000000u, 0x7540 + b));
}

__device__ __forceinline__ void accumulate_int4(const Packed<kINT4> &p, float (&acc)[32]) {
    const float s = __half2float(__ushort_as_half(p.scale));
    const float off = 8388608.0f + 8.0f;                            // 2^23 + bias
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = p.w[i] & 0x0F0F0F0Fu;                   // even elements
        const uint32_t hi = (p.w[i] >> 4) & 0x0F0F0F0Fu;            // odd elements
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float q0 = __fsub_rn(magic_code_to_float(lo, b), off);
            const float q1 = __fsub_rn(magic_code_to_float(hi, b), off);
            acc[8 * i + 2 * b] = __fmaf_rn(q0, s, acc[8 * i + 2 * b]);
            acc[8 * i + 2 * b + 1] = __fmaf_rn(q1, s, acc[8 * i + 2 * b + 1]);
        }
    }
}

// Four INT3 codes of elements 4g..4g+3, one per byte.
__device__ __forceinline__ uint32_t int3_codes4(const Packed<kINT3> &p, int g) {
    const uint32_t q2 = (p.q2w[g >> 2] >> (8 * (g & 3))) & 0xFFu;     // 4 x 2 bits
    uint32_t lo = q2 | (q2 << 6) | (q2 << 12) | (q2 << 18);           // field m -> byte m
    lo &= 0x03030303u;
    const uint32_t nib = (p.q1w >> (4 * g)) & 0xFu;                   // 4 x 1 bit
    const uint32_t hi = (nib * 0x00204081u) & 0x01010101u;            // bit m -> byte m
    return lo | (hi << 2);
}

__device__ __forceinline__ void accumulate_int3(const Packed<kINT3> &p, float (&acc)[32]) {
    const float s = __half2float(__ushort_as_half(p.scale));
    const float off = 8388608.0f + 4.0f;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const uint32_t c4 = int3_codes4(p, g);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float q = __fsub_rn(magic_code_to_float(c4, b), off);
            acc[4 * g + b] = __fmaf_rn(q, s, acc[4 * g + b]);
        }
    }
}

// FP8: v = fl32(e4m3(code) * s), then acc = fl32(acc + v) (two roundings, no FMA).
__device__ __forceinline__ void accumulate_fp8(const Packed<kFP8> &p, float (&acc)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float e0, e1;
            unpack_e4m3x2(p.w[i] >> (16 * h), e0, e1);
            const int j = 4 * i + 2 * h;
            acc[j] = __fadd_rn(acc[j], __fmul_rn(e0, p.scale));
            acc[j + 1] = __fadd_rn(acc[j + 1], __fmul_rn(e1, p.scale));
        }
    }
}

// ---------------------------------------------------------------------------
// Block encoders from binary32 values (used by stage 1 and stage 2).
// WANT_V additionally returns the decoded result of the block as BF16 pairs
// (the value the gathered wire decodes to), for the fused decode.
// ---------------------------------------------------------------------------
template <bool WANT_V>
__device__ __forceinline__ void encode_int4(const float (&x)[32], float a, Packed<kINT4> &p, uint32_t (&o)[16]) {
    const IntScale k = int_scale<4>(a);
    p.scale = k.bits;
    if (k.fast) int4_body<true, WANT_V>(x, k, p.w, o);
    else int4_body<false, WANT_V>(x, k, p.w, o);
}

template <bool WANT_V>
__device__ __forceinline__ void encode_int3(const float (&x)[32], float a, Packed<kINT3> &p, uint32_t (&o)[16]) {
    const IntScale k = int_scale<3>(a);
    p.scale = k.bits;
    if (k.fast) int3_body<true, WANT_V>(x, k, p.q2w, p.q1w, o);
    else int3_body<false, WANT_V>(x, k, p.q2w, p.q1w, o);
}

template <bool WANT_V>
__device__ __forceinline__ void encode_fp8(const float (&x)[32], float a, Packed<kFP8> &p, uint32_t (&o)[16]) {
    const float s = __fdiv_rn(a, 448.0f);
    if (!(s >= 1.17549435e-38f)) {                    // below 2^-126 (or zero): zero block
#pragma unroll
        for (int i = 0; i < 8; ++i) p.w[i] = 0u;
        p.scale = 0.f;
        if (WANT_V) {
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = 0u;
        }
        return;
    }
    const float inv = __frcp_rn(s);                   // fl32(1 / s)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = pack_e4m3x2(__fmul_rn(x[4 * i], inv), __fmul_rn(x[4 * i + 1], inv));
        const uint32_t hi = pack_e4m3x2(__fmul_rn(x[4 * i + 2], inv), __fmul_rn(x[4 * i + 3], inv));
        p.w[i] = lo | (hi << 16);
        if (WANT_V) {
            float e0, e1, e2, e3;
            unpack_e4m3x2(lo, e0, e1);
            unpack_e4m3x2(hi, e2, e3);
            o[2 * i] = pack_bf16x2(__fmul_rn(e0, s), __fmul_rn(e1, s));
            o[2 * i + 1] = pack_bf16x2(__fmul_rn(e2, s), __fmul_rn(e3, s));
        }
    }
    p.scale = s;
}

// Decode one block to BF16 (RNE), 16 packed words (element 2k in the low half).
// The value is q * s (one exact product), rounded once to BF16.
__device__ __forceinline__ void decode_int4(const Packed<kINT4> &p, uint32_t (&o)[16]) {
    const float s = __half2float(__ushort_as_half(p.scale));
    const float off = 8388608.0f + 8.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = p.w[i] & 0x0F0F0F0Fu;
        const uint32_t hi = (p.w[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float q0 = __fsub_rn(magic_code_to_float(lo, b), off);
            const float q1 = __fsub_rn(magic_code_to_float(hi, b), off);
            o[4 * i + b] = pack_bf16x2(__fmul_rn(q0, s), __fmul_rn(q1, s));
        }
    }
}

__device__ __forceinline__ void decode_int3(const Packed<kINT3> &p, uint32_t (&o)[16]) {
    const float s = __half2float(__ushort_as_half(p.scale));
    const float off = 8388608.0f + 4.0f;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const uint32_t c4 = int3_codes4(p, g);
        float q[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) q[b] = __fsub_rn(magic_code_to_float(c4, b), off);
        o[2 * g] = pack_bf16x2(__fmul_rn(q[0], s), __fmul_rn(q[1], s));
        o[2 * g + 1] = pack_bf16x2(__fmul_rn(q[2], s), __fmul_rn(q[3], s));
    }
}

__device__ __forceinline__ void decode_fp8(const Packed<kFP8> &p, uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float e0, e1;
            unpack_e4m3x2(p.w[i] >> (16 * h), e0, e1);
            o[2 * i + h] = pack_bf16x2(__fmul_rn(e0, p.scale), __fmul_rn(e1, p.scale));
        }
    }
}

}  // namespace lpar
