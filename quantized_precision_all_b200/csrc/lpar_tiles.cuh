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
#pragma once

#include "lpar.h"
#include "lpar_codec.cuh"

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

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
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

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
struct NoSink {
    __device__ __forceinline__ void put(int, uint4) const {}
};
struct StageSink {                                   // thread t's 64-B region of the stage
    uint8_t *stage;
    int t;
    __device__ __forceinline__ void put(int j, uint4 v) const {
        *reinterpret_cast<uint4 *>(stage + swz(t, j)) = v;
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
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void stage_load_chunk(uint8_t *stage, const uint8_t *src, int ntiles) {
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int g = t + kThreads * k;
        if (g < ntiles * 256) cp_async16(stage + swz(g >> 2, g & 3), src + 16 * (size_t)g);
    }
}

// ---------------------------------------------------------------------------
// Host-side helpers.
// ---------------------------------------------------------------------------
// Resident CTAs of a kernel on the current device (SM count x occupancy), cached
// per device and kernel; 0 when the query fails.
template <class K>
static unsigned resident_ctas(K kernel) {
    static std::atomic<unsigned> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    unsigned v = cache[dev].load(std::memory_order_relaxed);
    if (v) return v;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess) return 0;
    v = (unsigned)(sms * (per_sm > 0 ? per_sm : 1));
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

static inline bool codec_ok(int c) { return c >= LPAR_CODEC_BF16 && c <= LPAR_CODEC_MXFP4; }
static inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static inline lpar_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? LPAR_OK : LPAR_ERR_CUDA;
}

// Reduction of N ranks' messages to BF16 (stage 1, then the FP32 sum rounded
// once to BF16, no requantisation), defined in lpar_collectives.cu: into every
// out[r] (all = true: the one-shot all-reduce) or into the shard owners
// (all = false: the reduce-scatter).  `wire` holds N stage-1 wires (unused
// for BF16).
void launch_reduce_to_bf16(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N,
                           size_t tiles, bool all, cudaStream_t st);

}  // namespace lpar
