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
//   MXFP4:     ("Microscaling Data Formats for Deep Learning", abstract: a
//              scale shared by a block of narrow floating-point elements)
//              E = clamp(floor(log2(absmax)) - 2, -127, 127) stored as the E8M0
//              byte E + 127; code = e2m1_rne_satfinite(x / 2^E), sign kept.
//
// Exact RNE(x / s) without a per-element division
// -----------------------------------------------
// Fast path (normal, unsaturated binary16 scale, so |x/s| <= qmax(1 + 2^-11)):
// r approximates 1/s within 2^-23 (one hardware reciprocal), so the exact
// product x*r is within 7.01 * 2^-23 < 2^-20 of Q = x/s.  Three roundings,
// all FMAs on exact operands, give q:
//   C2 = fl(x*r + 2M)   (M = 1.5*2^23; 2M has ulp 2): 2M + 2*k2, 2*k2 = the even
//                        integer nearest to x*r;
//   f2 = fl(x*r - 2*k2)  in [-1, 1];
//   C3 = fl(f2*eta + (M + 2*k2)), eta = 1 - 2^-18 (ulp 1): M + q with
//        q = 2*k2 + RNE(f2 * eta).
// If Q is an exact tie m + 1/2, 2*k2 is the even one of m, m+1 and
// |f2| <= 1/2 + 2^-20, so |f2 * eta| < 1/2 and q = 2*k2 = RNE(Q).  Otherwise q
// is RNE(Q) unless Q lies within 2^-18 + 2^-20 of a half-integer on its odd
// side.  At stage 1 (BF16 x, 8-bit significand; binary16 s, 11 bits) a non-tie
// quotient is at least 1/(2S) > 2^-12 from a half-integer, so stage 1 is exact
// as it stands.  At stage 2 (binary32 sums) each q is verified: e = x - q*s is
// exact; a wrong q has |e| > s/2, and since e - (+-s/2) is a nonzero multiple
// of ulp(s/2) >= (s/2) 2^-24, e^2 - (s/2)^2 > (s/2)^2 2^-23 >= ulp((s/2)^2): the
// sign of e^2 - nextafter((s/2)^2) flags it, while an exact tie (|e| = s/2) and
// every correct q pass.  A flagged block (rare) is redone on the exact path.  Blocks with a subnormal, zero or saturated scale take the exact
// path.
//
// Exact path: k = RNE(fl(x*r) - 1/2) is RNE(x/s) or one less; the midpoint
// m = (k + 1/2) * s is exact in binary32 ((2k+1) has <= 5 bits, s <= 11 bits),
// so comparing x with m decides exactly: q = k + 1 when x > m, or when x == m
// and k is odd (ties to even); otherwise q = k.
//
// Scale: fl32(absmax / qmax) by Markstein's correction (IBM J. Res. Dev. 34,
// 1990): y = RN(1/qmax), q0 = RN(a*y), rem = fma(-q0, qmax, a) (exact),
// result = RN(q0 + rem*y).  For qmax = 7 and 3 this equals the IEEE quotient for
// every non-negative binary32 a (checked exhaustively on the host).
//
// Codes are packed with exact binary32 polynomials: for codes c_m of a group,
// Sum c_m 2^(w m) is formed by an FMA chain (< 2^24, exact) and added to M,
// which puts the packed bits in the low mantissa of the result.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace lpar {

constexpr int kBlock = 32;
constexpr int kTileElems = 2048;
constexpr int kBlocksPerTile = 64;

enum CodecId : int { kBF16 = 0, kFP8 = 1, kINT4 = 2, kINT3 = 3, kMXFP4 = 4 };

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
template <> struct Layout<kMXFP4> {
    static constexpr int kTileBytes = 1088, kScaleOff = 1024;
};
template <> struct Layout<kBF16> {
    static constexpr int kTileBytes = 4096;
};

// The packed payload of one block (codes + scale) as it sits in a tile.
template <int C> struct Packed;
template <> struct Packed<kINT4> { uint32_t w[4]; uint16_t scale; };          // 16 B codes
template <> struct Packed<kINT3> { uint32_t q2w[2]; uint32_t q1w; uint16_t scale; };
template <> struct Packed<kFP8> { uint32_t w[8]; float scale; };              // 32 B codes
template <> struct Packed<kMXFP4> { uint32_t w[4]; uint32_t scale; };         // 16 B codes, E8M0 byte

constexpr float kMagic = 12582912.0f;                 // 1.5 * 2^23: ulp 1, bits 0x4B400000
constexpr float kMagic2 = 25165824.0f;                // 3 * 2^23 = 1.5 * 2^24: ulp 2
constexpr float kEta = 1.0f - 0x1p-18f;               // shrinks exact ties below 1/2

// ---------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed binary32 pairs (sm_100 f32x2 arithmetic; each lane rounds like the
// scalar instruction, to nearest even, subnormals kept).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

// fl32(a * s + c) with a, s binary16 (the low or high half of a packed word):
// the product of two binary16 values is exact in binary32, so this rounds once.
__device__ __forceinline__ float fma_h(uint32_t a_pair, int hi, uint16_t s, float c) {
    float d;
    if (hi)
        asm("{.reg .f16 l, h, s;\n\tmov.b32 {l, h}, %1;\n\tmov.b16 s, %2;\n\t"
            "fma.rn.f32.f16 %0, h, s, %3;}" : "=f"(d) : "r"(a_pair), "h"(s), "f"(c));
    else
        asm("{.reg .f16 l, h, s;\n\tmov.b32 {l, h}, %1;\n\tmov.b16 s, %2;\n\t"
            "fma.rn.f32.f16 %0, l, s, %3;}" : "=f"(d) : "r"(a_pair), "h"(s), "f"(c));
    return d;
}

// Exact binary32 value of one half of a packed binary16 pair.
__device__ __forceinline__ float h2f(uint32_t pair, int hi) {
    return fma_h(pair, hi, 0x3C00u /* 1.0 */, -0.0f);
}

// Packed binary16 pair minus a packed constant (exact for the small integers used here).
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

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

// Packed E4M3x2 (16 bits) -> packed binary16 pair (exact: E4M3 is a subset of binary16).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)two));
    return h2;
}

// Two binary32 -> one byte of two E2M1 codes (RNE, finite saturation at +-6),
// `lo` in bits 0..3, zero-extended to 32 bits.
__device__ __forceinline__ uint32_t pack_e2m1x2(float lo, float hi) {
    uint32_t d;
    asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
        : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Eight binary32 -> eight E2M1 codes, element k in nibble k.
__device__ __forceinline__ uint32_t pack_e2m1x8(float a0, float a1, float a2, float a3, float a4, float a5,
                                                float a6, float a7) {
    const uint32_t b01 = __byte_perm(pack_e2m1x2(a0, a1), pack_e2m1x2(a2, a3), 0x0040);
    const uint32_t b23 = __byte_perm(pack_e2m1x2(a4, a5), pack_e2m1x2(a6, a7), 0x0040);
    return __byte_perm(b01, b23, 0x5410);
}

// Byte k of w (two E2M1 codes) -> packed binary16 pair (exact: E2M1 is a
// subset of binary16), the low nibble's element in the low half.  The byte is
// isolated first, so no other bits of the register reach the conversion.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t w, int k) {
    const uint32_t two = __byte_perm(w, 0u, 0x4440u + (uint32_t)k);
    uint32_t h;
    asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h) : "r"(two));
    return h;
}

// Eight E2M1 codes -> four packed binary16 pairs; pair j holds elements
// (2j, 2j + 1) in (low, high).
__device__ __forceinline__ void e2m1x8_to_h2(uint32_t w, uint32_t (&h)[4]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) h[k] = e2m1x2_to_h2(w, k);
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

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float absmax_f32x32(const float (&x)[32]) {
    float a[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) a[i] = max3(fabsf(x[3 * i]), fabsf(x[3 * i + 1]), fabsf(x[3 * i + 2]));
    a[10] = fmaxf(fabsf(x[30]), fabsf(x[31]));
    const float b0 = max3(a[0], a[1], a[2]), b1 = max3(a[3], a[4], a[5]);
    const float b2 = max3(a[6], a[7], a[8]), b3 = fmaxf(a[9], a[10]);
    return fmaxf(max3(b0, b1, b2), b3);
}

// ---------------------------------------------------------------------------
// INT4 / INT3 block scale.
// ---------------------------------------------------------------------------
struct IntScale {
    uint16_t bits;   // binary16 scale as stored in the tile
    float s;         // its value
    float r;         // fl(1/s), or 0 when s == 0
    float hs;        // s/2, or +inf when s == 0 (nothing ever rounds up)
    float lim;       // (qmax + 1) * s: bound applied on the exact path
    float t2;        // next binary32 above (s/2)^2: stage-2 verification threshold
    bool fast;       // normal, unsaturated scale: |x/s| <= qmax (1 + 2^-11), no clamp needed
};

// fl32(a / qmax), equal to the IEEE quotient (see the header comment).
template <int BITS>
__device__ __forceinline__ float div_qmax(float a) {
    constexpr float q = (float)((1 << (BITS - 1)) - 1);
    const float y = __uint_as_float(BITS == 4 ? 0x3E124925u : 0x3EAAAAABu);   // RN(1/7), RN(1/3)
    const float q0 = __fmul_rn(a, y);
    const float rem = __fmaf_rn(-q0, q, a);
    return __fmaf_rn(rem, y, q0);
}

// Hardware reciprocal, relative error below 2^-23.
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

template <int BITS>
__device__ __forceinline__ IntScale int_scale(float a) {
    constexpr int kQmax = (1 << (BITS - 1)) - 1;
    IntScale k;
    const float ratio = div_qmax<BITS>(a);
    uint16_t sb = __half_as_ushort(__float2half_rn(ratio));
    if (sb == 0x7C00u) sb = 0x7BFFu;                                   // saturate at 65504
    k.bits = sb;
    k.s = __half2float(__ushort_as_half(sb));
    k.fast = (sb >= 0x0400u) && (sb != 0x7BFFu);
    k.r = (k.s != 0.f) ? rcp_approx(k.s) : 0.f;
    k.hs = (k.s != 0.f) ? 0.5f * k.s : __int_as_float(0x7F800000);
    k.lim = (float)(kQmax + 1) * k.s;                                 // exact
    const float hs2 = __fmul_rn(0.5f * k.s, 0.5f * k.s);              // exact (11-bit s)
    k.t2 = __uint_as_float(__float_as_uint(hs2) + 1u);                // one ulp above
    return k;
}

// ---------------------------------------------------------------------------
// Exact path (any scale; used for flagged blocks).
// ---------------------------------------------------------------------------
template <int BITS, bool FAST, bool WANT_V>
__device__ __forceinline__ uint32_t int_code(float x, const IntScale &k, float &v) {
    constexpr int kQmax = (1 << (BITS - 1)) - 1;
    constexpr int kBias = 1 << (BITS - 1);
    const float magic = kMagic + (float)kBias;                        // 1.5 * 2^23 + bias
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

// ---------------------------------------------------------------------------
// Fast path.  Returns false when some element is near a tie (the caller then
// redoes the block on the exact path); outputs are only valid when true.
// ---------------------------------------------------------------------------

// One element pair -> C3 = M + BIAS + q (q = RNE(x/s), see the header comment;
// the offset BIAS is folded into the addend of the last step, which stays in
// [2^23, 2^24), so the rounding is unchanged) and, when needed, -q.
// STAGE2: clears bit 31 of `ok` when some q fails the exact verification.
template <bool STAGE2, bool WANT_NQ, int BIAS = 0>
__device__ __forceinline__ float2 round_pair_c(float2 xv, const IntScale &k, uint32_t &ok, float2 &nq) {
    const float2 r2 = splat(k.r), M4 = splat(kMagic2);
    const float2 C2 = fma2(xv, r2, M4);                // 2M + 2 k2 (exact product inside)
    const float2 nq2 = sub2(M4, C2);                   // -2 k2
    const float2 B = sub2(C2, splat(kMagic - (float)BIAS));   // M + BIAS + 2 k2
    const float2 f2 = fma2(xv, r2, nq2);               // x r - 2 k2
    const float2 C3 = fma2(f2, splat(kEta), B);        // M + BIAS + q
    if (WANT_NQ || STAGE2) nq = sub2(splat(kMagic + (float)BIAS), C3);   // -q (exact)
    if (STAGE2) {
        const float2 e = fma2(nq, splat(k.s), xv);     // x - q s, exact
        const float2 d = fma2(e, e, splat(-k.t2));     // < 0 iff |e| <= s/2
        ok &= __float_as_uint(d.x) & __float_as_uint(d.y);
    }
    return C3;
}

template <bool STAGE2>
__device__ __forceinline__ float2 round_pair(float2 xv, const IntScale &k, uint32_t &ok) {
    float2 nq;
    round_pair_c<STAGE2, true>(xv, k, ok, nq);
    return nq;
}

// INT4: lanes hold elements (8i + m, 8i + 4 + m); each lane packs 4 nibbles
// (16 bits) with Q = Sum_m (-q_m) 16^m, P = (M + 0x8888) - Q.
// Decoded values go to `sink.put(j, v0, ..., v7)`: piece j holds elements
// 8j..8j+7 in order, handed over as soon as they exist.
template <bool STAGE2, bool WANT_V, class Sink>
__device__ __forceinline__ bool int4_fast(const float (&x)[32], const IntScale &k, uint32_t (&w)[4],
                                          const Sink &sink) {
    const float2 ns2 = splat(-k.s), S16 = splat(16.f);
    uint32_t ok = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 nq[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) nq[m] = round_pair<STAGE2>(make_float2(x[8 * i + m], x[8 * i + 4 + m]), k, ok);
        float2 Q = fma2(nq[3], S16, nq[2]);
        Q = fma2(Q, S16, nq[1]);
        Q = fma2(Q, S16, nq[0]);
        const float2 P = sub2(splat(kMagic + 34952.0f), Q);     // 34952 = 0x8888: bias 8 per nibble
        w[i] = __byte_perm(__float_as_uint(P.x), __float_as_uint(P.y), 0x5410);
        if (WANT_V) {
            float2 v[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) v[m] = fma2(nq[m], ns2, splat(0.f));   // q s (+0 for q = 0)
            sink.put(i, v[0].x, v[1].x, v[2].x, v[3].x, v[0].y, v[1].y, v[2].y, v[3].y);
        }
    }
    return (ok >> 31) != 0u;
}

// INT3 from the integer bits of C3 = M + code (code = q + 4 in bits 0..2,
// since M = 0x4B400000 as bits): lanes hold elements (4g + i, 16 + 4g + i).
// PRMTs gather the code bytes of elements 4g..4g+3 into one word W_g, and two
// multiplies move its bit fields into place without carries (every cross
// term lands below the target byte, at distinct positions):
//   (W & 0x03030303) * 0x01041040: byte 3 = the four low-2-bit fields (q2w);
//   (W & 0x04040404) * 0x00408102: bits 24..27 = the four high bits (q1w),
//   or * 0x04081020 for bits 28..31, so two groups combine with one OR.
// Everything after the rounding runs on the integer ALU, not the FMA pipe.
__device__ __forceinline__ uint32_t code_bytes4(float a, float b, float c, float d) {
    return __byte_perm(__byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040),
                       __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040), 0x5410);
}

template <bool STAGE2, bool WANT_V, class Sink>
__device__ __forceinline__ bool int3_fast(const float (&x)[32], const IntScale &k, uint32_t (&q2w)[2],
                                          uint32_t &q1w, const Sink &sink) {
    const float2 ns2 = splat(-k.s);
    uint32_t ok = 0xFFFFFFFFu;
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int p = 0; p < 2; ++p) {                      // groups 2p, 2p+1: elements 8p..8p+7 and 16+8p..
        float2 v[8];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int g = 2 * p + gg;
            float2 C[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float2 nq;
                C[i] = round_pair_c<STAGE2, WANT_V, 4>(make_float2(x[4 * g + i], x[16 + 4 * g + i]), k, ok, nq);
                if (WANT_V) v[4 * gg + i] = fma2(nq, ns2, splat(0.f));   // q s (+0 for q = 0)
            }
            const uint32_t W0 = code_bytes4(C[0].x, C[1].x, C[2].x, C[3].x);   // elements 4g .. 4g+3
            const uint32_t W1 = code_bytes4(C[0].y, C[1].y, C[2].y, C[3].y);   // elements 16+4g ..
            lo[g] = (W0 & 0x03030303u) * 0x01041040u;
            lo[4 + g] = (W1 & 0x03030303u) * 0x01041040u;
            hi[g] = (W0 & 0x04040404u) * ((g & 1) ? 0x04081020u : 0x00408102u);
            hi[4 + g] = (W1 & 0x04040404u) * ((g & 1) ? 0x04081020u : 0x00408102u);
        }
        if (WANT_V) {                                  // piece j = elements 8j .. 8j+7
            sink.put(p, v[0].x, v[1].x, v[2].x, v[3].x, v[4].x, v[5].x, v[6].x, v[7].x);
            sink.put(2 + p, v[0].y, v[1].y, v[2].y, v[3].y, v[4].y, v[5].y, v[6].y, v[7].y);
        }
    }
    q2w[0] = __byte_perm(__byte_perm(lo[0], lo[1], 0x0073), __byte_perm(lo[2], lo[3], 0x0073), 0x5410);
    q2w[1] = __byte_perm(__byte_perm(lo[4], lo[5], 0x0073), __byte_perm(lo[6], lo[7], 0x0073), 0x5410);
    q1w = __byte_perm(__byte_perm(hi[0] | hi[1], hi[2] | hi[3], 0x0073),
                      __byte_perm(hi[4] | hi[5], hi[6] | hi[7], 0x0073), 0x5410);
    return (ok >> 31) != 0u;
}

// ---------------------------------------------------------------------------
// Block encoders from binary32 values (used by stage 1 and stage 2).
// WANT_V additionally returns the decoded result of the block as BF16 pairs
// (the value the gathered wire decodes to), for the fused decode.
// ---------------------------------------------------------------------------
// Out-of-line exact path.  It is rare (near ties at stage 2, subnormal or
// saturated scales), so it runs one element at a time from local memory with a
// rolled loop: few registers, so the hot path keeps a small register allocation.
template <int BITS, bool WANT_V>
__device__ __noinline__ void int_exact_codes(const float *x, IntScale k, uint8_t *code, float *v) {
#pragma unroll 1
    for (int j = 0; j < 32; ++j) {
        float vj = 0.f;
        const uint32_t c = k.fast ? int_code<BITS, true, WANT_V>(x[j], k, vj) : int_code<BITS, false, WANT_V>(x[j], k, vj);
        code[j] = (uint8_t)c;
        if (WANT_V) v[j] = vj;
    }
}

template <bool WANT_V, class Sink>
__device__ __forceinline__ void values_from_local(const float *v, const Sink &sink) {
    if (WANT_V) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            sink.put(j, v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3], v[8 * j + 4], v[8 * j + 5],
                     v[8 * j + 6], v[8 * j + 7]);
    }
}

__device__ __forceinline__ void pack_int4_local(const uint8_t *cs, Packed<kINT4> &p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) w |= (uint32_t)cs[8 * i + j] << (4 * j);
        p.w[i] = w;
    }
}

__device__ __forceinline__ void pack_int3_local(const uint8_t *cs, Packed<kINT3> &p) {
    uint32_t q2[2] = {0u, 0u}, q1 = 0u;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        q2[j >> 4] |= ((uint32_t)cs[j] & 3u) << (2 * (j & 15));
        q1 |= ((uint32_t)cs[j] >> 2) << j;
    }
    p.q2w[0] = q2[0];
    p.q2w[1] = q2[1];
    p.q1w = q1;
}

// Exact encoding of a block whose values are in local memory (rare path):
// scale, codes, packing and the decoded values.
template <int C, bool WANT_V, class Sink>
__device__ __forceinline__ void encode_int_exact_local(const float *xs, const IntScale &k, Packed<C> &p,
                                                       const Sink &sink) {
    float vs[32];
    uint8_t cs[32];
    int_exact_codes<Layout<C>::kBits, WANT_V>(xs, k, cs, vs);
    if constexpr (C == kINT4) pack_int4_local(cs, p);
    else pack_int3_local(cs, p);
    values_from_local<WANT_V>(vs, sink);
}

// Stage 1 (and any caller that keeps x): fast path, else copy x to local
// memory and take the exact path.
template <int C, bool STAGE2, bool WANT_V, class Sink>
__device__ __forceinline__ void encode_int(const float (&x)[32], float a, Packed<C> &p, const Sink &sink) {
    const IntScale k = int_scale<Layout<C>::kBits>(a);
    p.scale = k.bits;
    bool ok = k.fast;
    if constexpr (C == kINT4) {
        if (ok) ok = int4_fast<STAGE2, WANT_V>(x, k, p.w, sink);
    } else {
        if (ok) ok = int3_fast<STAGE2, WANT_V>(x, k, p.q2w, p.q1w, sink);
    }
    if (!ok) {
        float xs[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) xs[j] = x[j];
        encode_int_exact_local<C, WANT_V>(xs, k, p, sink);
    }
}

template <bool WANT_V, class Sink>
__device__ __forceinline__ void encode_fp8(const float (&x)[32], float a, Packed<kFP8> &p, const Sink &sink) {
    const float s = __fdiv_rn(a, 448.0f);
    if (!(s >= 1.17549435e-38f)) {                    // below 2^-126 (or zero): zero block
#pragma unroll
        for (int i = 0; i < 8; ++i) p.w[i] = 0u;
        p.scale = 0.f;
        if (WANT_V) {
#pragma unroll
            for (int j = 0; j < 4; ++j) sink.put(j, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
    const float inv = __frcp_rn(s);                   // fl32(1 / s)
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {                     // scalar IEEE products (subnormals kept)
        const uint32_t lo = pack_e4m3x2(__fmul_rn(x[4 * i], inv), __fmul_rn(x[4 * i + 1], inv));
        const uint32_t hi = pack_e4m3x2(__fmul_rn(x[4 * i + 2], inv), __fmul_rn(x[4 * i + 3], inv));
        p.w[i] = lo | (hi << 16);
        if (WANT_V) {                                 // scalar: e * s may be subnormal
            const uint32_t h0 = e4m3x2_to_h2(lo), h1 = e4m3x2_to_h2(hi);
            float *oi = o + 4 * (i & 1);
            oi[0] = __fmul_rn(h2f(h0, 0), s);
            oi[1] = __fmul_rn(h2f(h0, 1), s);
            oi[2] = __fmul_rn(h2f(h1, 0), s);
            oi[3] = __fmul_rn(h2f(h1, 1), s);
            if (i & 1) sink.put(i >> 1, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
        }
    }
    p.scale = s;
}

// MXFP4.  E8M0 scale byte ec = max(biased exponent of absmax - 2, 0): for a
// normal absmax the biased exponent is floor(log2 a) + 127, so ec = E + 127
// with E = floor(log2 a) - 2, and the clamp at 0 is E >= -127 (absmax zero or
// below 2^-125).  x / 2^E is the product with 2^-E = 2^(127 - ec), whose
// biased exponent 254 - ec is in [1, 254], so it is exact unless it falls
// below 2^-126, where every value rounds to a signed zero either way.  Scalar IEEE products keep
// subnormal inputs (stage-2 sums can be subnormal).
__device__ __forceinline__ uint32_t mx_scale_code(float a) {
    const int ef = (int)(__float_as_uint(a) >> 23);
    return (uint32_t)max(ef - 2, 0);
}
__device__ __forceinline__ float mx_scale_value(uint32_t ec) {       // 2^(ec - 127), exact
    return __uint_as_float(ec ? (ec << 23) : 0x00400000u);
}

template <bool WANT_V, class Sink>
__device__ __forceinline__ void encode_mxfp4(const float (&x)[32], float a, Packed<kMXFP4> &p, const Sink &sink) {
    const uint32_t ec = mx_scale_code(a);
    const float m = __uint_as_float((254u - ec) << 23);          // 2^-E
    p.scale = ec;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float *xi = x + 8 * i;
        p.w[i] = pack_e2m1x8(__fmul_rn(xi[0], m), __fmul_rn(xi[1], m), __fmul_rn(xi[2], m), __fmul_rn(xi[3], m),
                             __fmul_rn(xi[4], m), __fmul_rn(xi[5], m), __fmul_rn(xi[6], m), __fmul_rn(xi[7], m));
        if (WANT_V) {                                             // E2M1 value * 2^E: exact, so is its BF16
            const float sv = mx_scale_value(ec);
            uint32_t h[4];
            float o[8];
            e2m1x8_to_h2(p.w[i], h);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                o[2 * k] = __fmul_rn(h2f(h[k], 0), sv);
                o[2 * k + 1] = __fmul_rn(h2f(h[k], 1), sv);
            }
            sink.put(i, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
        }
    }
}

// ---------------------------------------------------------------------------
// Dequantisation.  INT codes become exact binary16 integers q (magic 1024 +
// code, minus 1024 + bias), and acc = fl32(acc + q*s) is one mixed-precision
// FMA with the binary16 scale: q*s is exact in binary32, so it rounds once,
// exactly like the definition's acc + (float)q * s.
// ---------------------------------------------------------------------------

// INT4 word (elements 8i..8i+7) -> four packed binary16 pairs of q:
// h[0] = (e0, e2), h[1] = (e4, e6), h[2] = (e1, e3), h[3] = (e5, e7).
__device__ __forceinline__ void int4_word_to_h2(uint32_t w, uint32_t (&h)[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint32_t bias = 0x64086408u;                 // (1032, 1032) in binary16
    h[0] = hsub2(__byte_perm(lo, 0x64646464u, 0x4140), bias);
    h[1] = hsub2(__byte_perm(lo, 0x64646464u, 0x4342), bias);
    h[2] = hsub2(__byte_perm(hi, 0x64646464u, 0x4140), bias);
    h[3] = hsub2(__byte_perm(hi, 0x64646464u, 0x4342), bias);
}

// INT3 half-block (elements 16*half .. 16*half+15) -> eight packed binary16
// pairs of q.  Codes are assembled one per nibble: the low two bits of the
// even (odd) elements are q2w & 0x33333333 ((q2w >> 2) & 0x33333333).  The
// sixteen q1w bits of the half are spread to every second bit (bit j -> bit
// 2j), which puts the bit of element 2k at 4k and that of element 2k + 1 at
// 4k + 2: the odd elements' high bits are then in place, the even elements'
// two bits to the left.  A nibble code c (0..7) indexes an 8-byte table with
// one PRMT: the binary16 value of q = c - 4 is -4, -3, ..., 3, whose low byte
// is always 0, so the table holds only the high bytes and two more PRMTs
// interleave zero bytes.
// h[0..3] = (e0,e2) (e4,e6) (e8,e10) (e12,e14); h[4..7] = (e1,e3) (e5,e7)
// (e9,e11) (e13,e15), indices relative to 16*half.
__device__ __forceinline__ uint32_t spread_half_bits(uint32_t q1w, int half) {   // bit 16*half + j -> bit 2j
    uint32_t t = __byte_perm(q1w, 0u, half ? 0x4342 : 0x4140);              // byte k -> byte 2k
    t = (t | (t << 4)) & 0x0F0F0F0Fu;
    t = (t | (t << 2)) & 0x33333333u;
    return (t | (t << 1)) & 0x55555555u;
}

__device__ __forceinline__ void int3_half_to_h2(const Packed<kINT3> &p, int half, uint32_t (&h)[8]) {
    const uint32_t w = p.q2w[half];
    const uint32_t d = spread_half_bits(p.q1w, half);
    const uint32_t ce = (w & 0x33333333u) | ((d << 2) & 0xCCCCCCCCu);        // even elements
    const uint32_t co = ((w >> 2) & 0x33333333u) | (d & 0xCCCCCCCCu);        // odd elements
    const uint32_t T0 = 0xBCC0C2C4u;       // high bytes of -1, -2, -3, -4 (codes 3..0)
    const uint32_t T1 = 0x42403C00u;       // high bytes of  3,  2,  1,  0 (codes 7..4)
    const uint32_t e0 = __byte_perm(T0, T1, ce), e1 = __byte_perm(T0, T1, ce >> 16);
    const uint32_t o0 = __byte_perm(T0, T1, co), o1 = __byte_perm(T0, T1, co >> 16);
    h[0] = __byte_perm(e0, 0u, 0x1404);
    h[1] = __byte_perm(e0, 0u, 0x3424);
    h[2] = __byte_perm(e1, 0u, 0x1404);
    h[3] = __byte_perm(e1, 0u, 0x3424);
    h[4] = __byte_perm(o0, 0u, 0x1404);
    h[5] = __byte_perm(o0, 0u, 0x3424);
    h[6] = __byte_perm(o1, 0u, 0x1404);
    h[7] = __byte_perm(o1, 0u, 0x3424);
}

__device__ __forceinline__ void accumulate_int4(const Packed<kINT4> &p, float (&acc)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h[4];
        int4_word_to_h2(p.w[i], h);
        acc[8 * i + 0] = fma_h(h[0], 0, p.scale, acc[8 * i + 0]);
        acc[8 * i + 2] = fma_h(h[0], 1, p.scale, acc[8 * i + 2]);
        acc[8 * i + 4] = fma_h(h[1], 0, p.scale, acc[8 * i + 4]);
        acc[8 * i + 6] = fma_h(h[1], 1, p.scale, acc[8 * i + 6]);
        acc[8 * i + 1] = fma_h(h[2], 0, p.scale, acc[8 * i + 1]);
        acc[8 * i + 3] = fma_h(h[2], 1, p.scale, acc[8 * i + 3]);
        acc[8 * i + 5] = fma_h(h[3], 0, p.scale, acc[8 * i + 5]);
        acc[8 * i + 7] = fma_h(h[3], 1, p.scale, acc[8 * i + 7]);
    }
}

__device__ __forceinline__ void accumulate_int3(const Packed<kINT3> &p, float (&acc)[32]) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t h[8];
        int3_half_to_h2(p, half, h);
        float *a = acc + 16 * half;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            a[4 * g + 0] = fma_h(h[g], 0, p.scale, a[4 * g + 0]);
            a[4 * g + 2] = fma_h(h[g], 1, p.scale, a[4 * g + 2]);
            a[4 * g + 1] = fma_h(h[4 + g], 0, p.scale, a[4 * g + 1]);
            a[4 * g + 3] = fma_h(h[4 + g], 1, p.scale, a[4 * g + 3]);
        }
    }
}

// FP8: v = fl32(e4m3(code) * s), then acc = fl32(acc + v) (two roundings, no FMA).
// Scalar IEEE operations: e * s can be subnormal (s may be as small as 2^-126),
// and the packed f32x2 forms are not relied on for subnormal results.
__device__ __forceinline__ void accumulate_fp8(const Packed<kFP8> &p, float (&acc)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t e = e4m3x2_to_h2(p.w[i] >> (16 * h));
            const int j = 4 * i + 2 * h;
            acc[j] = __fadd_rn(acc[j], __fmul_rn(h2f(e, 0), p.scale));
            acc[j + 1] = __fadd_rn(acc[j + 1], __fmul_rn(h2f(e, 1), p.scale));
        }
    }
}

// MXFP4: acc = fl32(acc + e * 2^E) in one FMA; the product has at most two
// significant bits and is at least 2^-128, so it is exact and the FMA rounds
// once, like the definition's acc + v.  Scalar: the product can be subnormal.
__device__ __forceinline__ void accumulate_mxfp4(const Packed<kMXFP4> &p, float (&acc)[32]) {
    const float sv = mx_scale_value(p.scale);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h[4];
        e2m1x8_to_h2(p.w[i], h);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 8 * i + 2 * k;
            acc[j] = __fmaf_rn(h2f(h[k], 0), sv, acc[j]);
            acc[j + 1] = __fmaf_rn(h2f(h[k], 1), sv, acc[j + 1]);
        }
    }
}

// Decode one block to BF16 (RNE), 16 packed words (element 2k in the low half).
// The value is q * s (one exact product; -0 addend keeps the product's zero sign).
__device__ __forceinline__ void decode_int4(const Packed<kINT4> &p, uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h[4];
        int4_word_to_h2(p.w[i], h);
        float v[8];
        v[0] = fma_h(h[0], 0, p.scale, -0.0f);
        v[2] = fma_h(h[0], 1, p.scale, -0.0f);
        v[4] = fma_h(h[1], 0, p.scale, -0.0f);
        v[6] = fma_h(h[1], 1, p.scale, -0.0f);
        v[1] = fma_h(h[2], 0, p.scale, -0.0f);
        v[3] = fma_h(h[2], 1, p.scale, -0.0f);
        v[5] = fma_h(h[3], 0, p.scale, -0.0f);
        v[7] = fma_h(h[3], 1, p.scale, -0.0f);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[4 * i + q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
    }
}

__device__ __forceinline__ void decode_int3(const Packed<kINT3> &p, uint32_t (&o)[16]) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t h[8];
        int3_half_to_h2(p, half, h);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            o[8 * half + 2 * g] = pack_bf16x2(fma_h(h[g], 0, p.scale, -0.0f), fma_h(h[4 + g], 0, p.scale, -0.0f));
            o[8 * half + 2 * g + 1] = pack_bf16x2(fma_h(h[g], 1, p.scale, -0.0f), fma_h(h[4 + g], 1, p.scale, -0.0f));
        }
    }
}

__device__ __forceinline__ void decode_fp8(const Packed<kFP8> &p, uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t e = e4m3x2_to_h2(p.w[i] >> (16 * h));
            o[2 * i + h] = pack_bf16x2(__fmul_rn(h2f(e, 0), p.scale), __fmul_rn(h2f(e, 1), p.scale));
        }
    }
}

__device__ __forceinline__ void decode_mxfp4(const Packed<kMXFP4> &p, uint32_t (&o)[16]) {
    const float sv = mx_scale_value(p.scale);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h[4];
        e2m1x8_to_h2(p.w[i], h);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            o[4 * i + k] = pack_bf16x2(__fmul_rn(h2f(h[k], 0), sv), __fmul_rn(h2f(h[k], 1), sv));
    }
}

}  // namespace lpar
