// lpar_tiles.cuh -- tile I/O, shared-memory staging and launch helpers shared
// by the all-reduce kernels (lpar_kernels.cu) and the standalone collectives
// (lpar_collectives.cu).  Device code plus a few host-side helpers.
//
// Work decomposition used throughout: a CTA of 256 threads owns 4 consecutive
// tiles; thread t owns block (t mod 64) of tile (t / 64), i.e. 32 consecutive
// elements.  Codes and scales of one warp's 32 blocks are contiguous in a tile,
// so packed loads/stores are coalesced as they are.  The BF16 side (64 B per
// thread) is staged through shared memory with an XOR swizzle so both the
// coalesced global access and the per-thread 64-B access are bank-conflict free.
// The warp-local kernels stage per warp: warp w copies, reads and stores only
// its half tile (bytes [2048w, 2048w + 2048) of a stage).
#pragma once

#include "lpar.h"
#include "lpar_codec.cuh"

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#ifndef LPAR_API
#define LPAR_API extern "C" __attribute__((visibility("default")))
#endif

namespace lpar {

constexpr int kThreads = 256;
constexpr int kTilesPerCta = kThreads / kBlocksPerTile;     // 4
constexpr int kStageBytes = kThreads * 64;                  // 16 KiB of BF16 per CTA
constexpr int kMaxRanks = LPAR_MAX_RANKS;
constexpr int kMaxDevices = 64;
constexpr size_t kMaxTiles = (size_t)1 << 33;               // 2^44 elements per rank: chunk indices fit 32 bits

struct InPtrs { const uint8_t *p[kMaxRanks]; };
struct OutPtrs { uint8_t *p[kMaxRanks]; };

// Byte offset of 16-B piece j (0..3) of thread t's 64-B block in the stage.
__device__ __forceinline__ int swz(int t, int j) { return 64 * t + 16 * (j ^ ((t >> 1) & 3)); }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

// Bulk asynchronous copies from shared to global memory, done by the TMA engine
// (no tensor map: both addresses 16-B aligned, a multiple of 16 bytes).  Each
// issuing thread tracks its own groups: commit after its copies, wait_read<K>
// before the shared source is rewritten (at most K newest groups still read
// it), and wait_read<0> before the CTA exits, since its shared memory is then
// released; the global writes themselves are complete when the grid is.
// Shared-memory writes of the generic proxy reach the copies through
// fence_async_smem() and a barrier.
__device__ __forceinline__ void bulk_store(void *gmem, const void *smem, unsigned bytes) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem), "r"(s), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int K>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(K) : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Packed block <-> tile bytes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_block(const uint8_t *tile, int b, Packed<kINT4> &p) {
    const uint4 c = *reinterpret_cast<const uint4 *>(tile + 16 * b);
    p.w[0] = c.x; p.w[1] = c.y; p.w[2] = c.z; p.w[3] = c.w;
    p.scale = *reinterpret_cast<const uint16_t *>(tile + Layout<kINT4>::kScaleOff + 2 * b);
}
__device__ __forceinline__ void store_block(uint8_t *tile, int b, const Packed<kINT4> &p) {
    *reinterpret_cast<uint4 *>(tile + 16 * b) = make_uint4(p.w[0], p.w[1], p.w[2], p.w[3]);
    *reinterpret_cast<uint16_t *>(tile + Layout<kINT4>::kScaleOff + 2 * b) = p.scale;
}
__device__ __forceinline__ void load_block(const uint8_t *tile, int b, Packed<kINT3> &p) {
    const uint2 c = *reinterpret_cast<const uint2 *>(tile + 8 * b);
    p.q2w[0] = c.x; p.q2w[1] = c.y;
    p.q1w = *reinterpret_cast<const uint32_t *>(tile + Layout<kINT3>::kQ1wOff + 4 * b);
    p.scale = *reinterpret_cast<const uint16_t *>(tile + Layout<kINT3>::kScaleOff + 2 * b);
}
__device__ __forceinline__ void store_block(uint8_t *tile, int b, const Packed<kINT3> &p) {
    *reinterpret_cast<uint2 *>(tile + 8 * b) = make_uint2(p.q2w[0], p.q2w[1]);
    *reinterpret_cast<uint32_t *>(tile + Layout<kINT3>::kQ1wOff + 4 * b) = p.q1w;
    *reinterpret_cast<uint16_t *>(tile + Layout<kINT3>::kScaleOff + 2 * b) = p.scale;
}
// FP8 codes: two 16-B accesses (the ABI guarantees 16-B alignment only).
__device__ __forceinline__ void load_block(const uint8_t *tile, int b, Packed<kFP8> &p) {
    const uint4 c0 = *reinterpret_cast<const uint4 *>(tile + 32 * b);
    const uint4 c1 = *reinterpret_cast<const uint4 *>(tile + 32 * b + 16);
    p.w[0] = c0.x; p.w[1] = c0.y; p.w[2] = c0.z; p.w[3] = c0.w;
    p.w[4] = c1.x; p.w[5] = c1.y; p.w[6] = c1.z; p.w[7] = c1.w;
    p.scale = *reinterpret_cast<const float *>(tile + Layout<kFP8>::kScaleOff + 4 * b);
}
__device__ __forceinline__ void store_block(uint8_t *tile, int b, const Packed<kFP8> &p) {
    *reinterpret_cast<uint4 *>(tile + 32 * b) = make_uint4(p.w[0], p.w[1], p.w[2], p.w[3]);
    *reinterpret_cast<uint4 *>(tile + 32 * b + 16) = make_uint4(p.w[4], p.w[5], p.w[6], p.w[7]);
    *reinterpret_cast<float *>(tile + Layout<kFP8>::kScaleOff + 4 * b) = p.scale;
}

__device__ __forceinline__ void load_block(const uint8_t *tile, int b, Packed<kMXFP4> &p) {
    const uint4 c = *reinterpret_cast<const uint4 *>(tile + 16 * b);
    p.w[0] = c.x; p.w[1] = c.y; p.w[2] = c.z; p.w[3] = c.w;
    p.scale = tile[Layout<kMXFP4>::kScaleOff + b];
}
__device__ __forceinline__ void store_block(uint8_t *tile, int b, const Packed<kMXFP4> &p) {
    *reinterpret_cast<uint4 *>(tile + 16 * b) = make_uint4(p.w[0], p.w[1], p.w[2], p.w[3]);
    tile[Layout<kMXFP4>::kScaleOff + b] = (uint8_t)p.scale;
}

// Destinations for the decoded BF16 words of a block (piece j = 16 B).
// ---------------------------------------------------------------------------
// binary32 messages: 128 B per thread (its 32-element block), eight 16-B
// pieces, swizzled as piece j of thread t at 128 t + 16 (j ^ (t & 7)): a
// warp's coalesced 16-B accesses (four threads' blocks) and its per-thread
// accesses (one piece of 32 threads) both spread over all eight 16-B bank
// groups, four accesses each.  A 4-tile chunk is 32 KiB.
// ---------------------------------------------------------------------------
constexpr int kStageBytesF32 = kThreads * 128;

__device__ __forceinline__ int swz32(int t, int j) { return 128 * t + 16 * (j ^ (t & 7)); }

__device__ __forceinline__ void stage_load_chunk_f32(uint8_t *stage, const uint8_t *src, int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int g = t + kThreads * k;                 // 16-B piece of the chunk (512 per tile)
        if (g < ntiles * 512) cp_async16(stage + swz32(g >> 3, g & 7), src + 16 * (size_t)g);
    }
}

__device__ __forceinline__ void stage_read_f32(const uint8_t *stage, int t, float (&x)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 q = *reinterpret_cast<const float4 *>(stage + swz32(t, j));
        x[4 * j] = q.x; x[4 * j + 1] = q.y; x[4 * j + 2] = q.z; x[4 * j + 3] = q.w;
    }
}

__device__ __forceinline__ void stage_to_outputs_f32(const uint8_t *stage, const OutPtrs &out, int N, size_t byte0,
                                                     int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int g = t + kThreads * k;
        if (g < ntiles * 512) {
            const uint4 d = *reinterpret_cast<const uint4 *>(stage + swz32(g >> 3, g & 7));
#pragma unroll
            for (int r = 0; r < kMaxRanks; ++r)
                if (r < N) *reinterpret_cast<uint4 *>(out.p[r] + byte0 + 16 * (size_t)g) = d;
        }
    }
}

// Destinations of the decoded values of a block: put(j, v0..v7) receives
// elements 8j..8j+7 (binary32, exact dequantised values).
struct NoSink {
    __device__ __forceinline__ void put(int, float, float, float, float, float, float, float, float) const {}
};
struct StageSink {                                   // BF16 (RNE) into thread t's 64-B region of the stage
    uint8_t *stage;
    int t;
    __device__ __forceinline__ void put(int j, float a0, float a1, float a2, float a3, float a4, float a5, float a6,
                                        float a7) const {
        *reinterpret_cast<uint4 *>(stage + swz(t, j)) =
            make_uint4(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3), pack_bf16x2(a4, a5), pack_bf16x2(a6, a7));
    }
};

struct StageSinkLinear {                             // BF16 (RNE), thread t's 64-B region in element order
    uint8_t *stage;                                  // (the layout a bulk copy sends as it is)
    int t;
    __device__ __forceinline__ void put(int j, float a0, float a1, float a2, float a3, float a4, float a5, float a6,
                                        float a7) const {
        *reinterpret_cast<uint4 *>(stage + 64 * t + 16 * j) =
            make_uint4(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3), pack_bf16x2(a4, a5), pack_bf16x2(a6, a7));
    }
};

struct StageSinkF32 {                                // binary32 into thread t's 128-B region
    uint8_t *stage;
    int t;
    __device__ __forceinline__ void put(int j, float a0, float a1, float a2, float a3, float a4, float a5, float a6,
                                        float a7) const {
        *reinterpret_cast<float4 *>(stage + swz32(t, 2 * j)) = make_float4(a0, a1, a2, a3);
        *reinterpret_cast<float4 *>(stage + swz32(t, 2 * j + 1)) = make_float4(a4, a5, a6, a7);
    }
};

template <int C, bool STAGE2, bool WANT_V, class Sink>
__device__ __forceinline__ void encode(const float (&x)[32], float a, Packed<C> &p, const Sink &sink) {
    if constexpr (C == kFP8) encode_fp8<WANT_V>(x, a, p, sink);
    else if constexpr (C == kMXFP4) encode_mxfp4<WANT_V>(x, a, p, sink);
    else encode_int<C, STAGE2, WANT_V>(x, a, p, sink);
}

template <int C>
__device__ __forceinline__ void accumulate(const Packed<C> &p, float (&acc)[32]) {
    if constexpr (C == kINT4) accumulate_int4(p, acc);
    else if constexpr (C == kINT3) accumulate_int3(p, acc);
    else if constexpr (C == kMXFP4) accumulate_mxfp4(p, acc);
    else accumulate_fp8(p, acc);
}

template <int C>
__device__ __forceinline__ void decode(const Packed<C> &p, uint32_t (&o)[16]) {
    if constexpr (C == kINT4) decode_int4(p, o);
    else if constexpr (C == kINT3) decode_int3(p, o);
    else if constexpr (C == kMXFP4) decode_mxfp4(p, o);
    else decode_fp8(p, o);
}

// Stage-2 rare path: recompute the block's FP32 sums from the N wires (same
// arithmetic, so the same values) and requantise it exactly, one element at a
// time.  Re-reading the wires lets the hot path drop the sums as it goes.
template <int C, bool WANT_V, class Sink>
__device__ __noinline__ void reduce_block_exact(const uint8_t *const *wp, int N, size_t tile, int b, Packed<C> *g,
                                                Sink sink) {
    constexpr int kBits = Layout<C>::kBits;
    constexpr int kBias = 1 << (kBits - 1);
    float acc[32];
#pragma unroll 1
    for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
#pragma unroll 1
    for (int r = 0; r < N; ++r) {
        const uint8_t *tb = wp[r] + tile * Layout<C>::kTileBytes;
        const float s = __half2float(__ushort_as_half(
            *reinterpret_cast<const uint16_t *>(tb + Layout<C>::kScaleOff + 2 * b)));
#pragma unroll 1
        for (int j = 0; j < 32; ++j) {
            int code;
            if constexpr (C == kINT4) {
                code = (tb[16 * b + j / 2] >> (4 * (j & 1))) & 0xF;
            } else {
                code = ((tb[8 * b + j / 4] >> (2 * (j & 3))) & 3) |
                       (((tb[Layout<kINT3>::kQ1wOff + 4 * b + j / 8] >> (j & 7)) & 1) << 2);
            }
            acc[j] = __fadd_rn(acc[j], __fmul_rn((float)(code - kBias), s));   // exact product
        }
    }
    float a = 0.f;
#pragma unroll 1
    for (int j = 0; j < 32; ++j) a = fmaxf(a, fabsf(acc[j]));
    const IntScale k = int_scale<kBits>(a);
    g->scale = k.bits;
    encode_int_exact_local<C, WANT_V>(acc, k, *g, sink);
}

// Stage 2 for one block: thread-owned block b of `tile`, N wires -> gathered
// wire (and the decoded BF16 words into `sink`).
template <int C, int N, bool WANT_V, class Sink>
__device__ __forceinline__ void reduce_block(const uint8_t *const *wp, size_t tile, int b, uint8_t *gather,
                                             const Sink &sink) {
    Packed<C> p[N];
#pragma unroll
    for (int r = 0; r < N; ++r) load_block(wp[r] + tile * Layout<C>::kTileBytes, b, p[r]);
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.0f;          // +0.0f, then ranks in ascending order
#pragma unroll
    for (int r = 0; r < N; ++r) accumulate<C>(p[r], acc);
    const float a = absmax_f32x32(acc);
    Packed<C> g;
    if constexpr (C == kFP8) {
        encode_fp8<WANT_V>(acc, a, g, sink);
    } else if constexpr (C == kMXFP4) {
        encode_mxfp4<WANT_V>(acc, a, g, sink);
    } else {
        const IntScale k = int_scale<Layout<C>::kBits>(a);
        g.scale = k.bits;
        bool ok = k.fast;
        if constexpr (C == kINT4) {
            if (ok) ok = int4_fast<true, WANT_V>(acc, k, g.w, sink);
        } else {
            if (ok) ok = int3_fast<true, WANT_V>(acc, k, g.q2w, g.q1w, sink);
        }
        if (!ok) reduce_block_exact<C, WANT_V>(wp, N, tile, b, &g, sink);
    }
    store_block(gather + tile * Layout<C>::kTileBytes, b, g);
}

// Thread t's 64-B BF16 block <-> the swizzled stage.
__device__ __forceinline__ void stage_read(const uint8_t *stage, int t, uint32_t (&w)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 q = *reinterpret_cast<const uint4 *>(stage + swz(t, j));
        w[4 * j] = q.x; w[4 * j + 1] = q.y; w[4 * j + 2] = q.z; w[4 * j + 3] = q.w;
    }
}
__device__ __forceinline__ void stage_write(uint8_t *stage, int t, const uint32_t (&w)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(stage + swz(t, j)) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// Coalesced copy of the staged BF16 chunk: tile k (k < ntiles) to dst[k].
__device__ __forceinline__ void stage_to_tile_dsts(const uint8_t *stage, uint8_t *const *dst, int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < kTilesPerCta; ++k) {
        if (k < ntiles) {
            const int g = t + kThreads * k;             // piece t of tile k
            *reinterpret_cast<uint4 *>(dst[k] + 16 * (size_t)t) =
                *reinterpret_cast<const uint4 *>(stage + swz(g >> 2, g & 3));
        }
    }
}

// Coalesced copy of the staged BF16 chunk (ntiles tiles) to N outputs.
__device__ __forceinline__ void stage_to_outputs(const uint8_t *stage, const OutPtrs &out, int N,
                                                 size_t byte0, int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int g = t + kThreads * k;                 // 16-B piece index in the chunk
        if (g < ntiles * 256) {
            const uint4 d = *reinterpret_cast<const uint4 *>(stage + swz(g >> 2, g & 3));
#pragma unroll
            for (int r = 0; r < kMaxRanks; ++r)
                if (r < N) *reinterpret_cast<uint4 *>(out.p[r] + byte0 + 16 * (size_t)g) = d;
        }
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_groups() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void stage_load_chunk(uint8_t *stage, const uint8_t *src, int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int g = t + kThreads * k;
        if (g < ntiles * 256) cp_async16(stage + swz(g >> 2, g & 3), src + 16 * (size_t)g);
    }
}

// Warp-local staging.  Warp w of a CTA owns blocks 32w .. 32w + 31 of the
// chunk (half of tile w / 2): bytes [2048w, 2048w + 2048) of a 16-KiB stage.
// Its lanes copy exactly those bytes (lane l: 16-B pieces 128w + l + 32k,
// k = 0..3, so every copy instruction of the warp covers 512 contiguous
// bytes), read only them and send only them, so the warp needs no barrier
// with the other warps: __syncwarp orders its lanes' accesses.
constexpr int kWarpBytes = 2048;

__device__ __forceinline__ void warp_load(uint8_t *stage, const uint8_t *chunk_src, int w, int lane) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int g = 128 * w + lane + 32 * k;
        cp_async16(stage + swz(g >> 2, g & 3), chunk_src + 16 * (size_t)g);
    }
}

// The warp's 2 KiB of a swizzled BF16 stage to every output at byte0.
__device__ __forceinline__ void warp_to_outputs(const uint8_t *stage, const OutPtrs &out, int N, size_t byte0, int w,
                                                int lane) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int g = 128 * w + lane + 32 * k;
        const uint4 d = *reinterpret_cast<const uint4 *>(stage + swz(g >> 2, g & 3));
#pragma unroll
        for (int r = 0; r < kMaxRanks; ++r)
            if (r < N) *reinterpret_cast<uint4 *>(out.p[r] + byte0 + 16 * (size_t)g) = d;
    }
}

// The warp's 2 KiB of a swizzled BF16 stage to one destination (the warp's
// half tile there).
__device__ __forceinline__ void warp_to_dst(const uint8_t *stage, uint8_t *dst, int w, int lane) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = lane + 32 * k, g = 128 * w + q;
        *reinterpret_cast<uint4 *>(dst + 16 * (size_t)q) = *reinterpret_cast<const uint4 *>(stage + swz(g >> 2, g & 3));
    }
}

// The rank-parallel tile forms (one tile per CTA, the N ranks' stage 1 spread
// over the CTA's threads) run up to 256 tiles per rank (1 MiB of BF16), 512
// for FP8 (measured on B200 with the forms timed alternately in one process,
// calls back to back and single: the all-reduce 25-48% faster at 128 KiB per
// rank for N = 2..8, 11-35% at 1 MiB; from 2 MiB per rank slower for every
// codec but FP8, which turns at 4 MiB).
template <int C>
__host__ __device__ constexpr size_t kTileFormMaxTiles() { return C == kFP8 ? 512 : 256; }

// ---------------------------------------------------------------------------
// Host-side helpers.
// ---------------------------------------------------------------------------
// Resident CTAs of a kernel on the current device (SM count x occupancy at
// `smem` bytes of dynamic shared memory), cached per device and per kernel
// (the template argument is the kernel itself, so every kernel has its own
// cache); 0 when the query fails.
template <auto Kernel>
static unsigned resident_ctas(int smem = 0) {
    static std::atomic<unsigned> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    unsigned v = cache[dev].load(std::memory_order_relaxed);
    if (v) return v;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, Kernel, kThreads, smem) != cudaSuccess) return 0;
    v = (unsigned)(sms * (per_sm > 0 ? per_sm : 1));
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

// SM count of the current device, cached per device; 0 when the query fails.
static inline unsigned sm_count() {
    static std::atomic<unsigned> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    unsigned v = cache[dev].load(std::memory_order_relaxed);
    if (v) return v;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 0;
    cache[dev].store((unsigned)sms, std::memory_order_relaxed);
    return (unsigned)sms;
}

// The opt-in to more than 48 KiB of dynamic shared memory, made once per
// device and per kernel; false when it fails.
template <auto Kernel>
static bool allow_dynamic_smem(int bytes) {
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    if (done[dev].load(std::memory_order_relaxed)) return true;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done[dev].store(1, std::memory_order_relaxed);
    return true;
}

static inline bool codec_ok(int c) { return c >= LPAR_CODEC_BF16 && c <= LPAR_CODEC_MXFP4; }
static inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around one C ABI call (host-side enqueue), for profilers that
// record NVTX; without an attached tool it costs a predicted branch.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

static inline lpar_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? LPAR_OK : LPAR_ERR_CUDA;
}

// Reduction of N ranks' messages to BF16 (stage 1, then the FP32 sum rounded
// once to BF16, no requantisation), defined in lpar_collectives.cu: into every
// out[r] (all = true: the one-shot all-reduce) or into the shard owners
// (all = false: the reduce-scatter).  `wire` holds N stage-1 wires (unused
// for BF16).  False when the launch could not be configured.
bool launch_reduce_to_bf16(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N,
                           size_t tiles, bool all, cudaStream_t st);

}  // namespace lpar
