// lpar_peer.cu -- the two-shot compressed all-reduce as one kernel per rank
// over peer memory, and the calls that share its buffers between processes.
//
// "RCCLX: Innovating GPU communications on AMD platforms", Direct Data Access:
// ranks move data by storing straight into each other's memory rather than
// through a separate collective library, and the tree all-reduce is a
// reduce-scatter followed by an all-gather; Low-Precision Collectives: what
// crosses the links is the quantised wire, the sums are formed in FP32.  One
// launch per rank runs three phases, with the exchange folded into them:
//   phase A  stage 1 of this rank's message.  Each wire tile is stored straight
//            into the mailbox of its shard's owner (slot = this rank; staged in
//            shared memory first when the owner is on another GPU, so that
//            the link carries whole 16-B stores); when a chunk of tiles is
//            there, a flag in the owner's memory is raised.
//   phase B  stage 2 of this rank's own shard.  Per chunk: wait for the chunk's
//            flag from every rank, sum the N wires in FP32 in ascending rank
//            order from +0, requantise, store the reduced tiles into every
//            rank's gathered wire and raise a flag in each rank's memory.
//   phase C  stage 3.  Per chunk of every shard: wait for its flag, decode the
//            gathered tiles into this rank's BF16 output.
// Tile by tile the arithmetic is that of lpar_allreduce (the same shard
// partition, the same rank order, the same requantisation), so the results
// are identical bit for bit.
//
// Geometry.  T tiles per rank; shard j = tiles [jT/N, (j+1)T/N); every shard
// is cut into P chunks (chunk c of shard j = its tiles [cS/P, (c+1)S/P), S the
// shard's size), P = min(ceil(ceil(T/N) / chunk), 1024) for the chunk size of
// peer_chunks (1 to 16 tiles by the message size), so every rank derives the
// same chunks from (N, T) alone.  Rank j's mailbox holds N slots of
// ceil(T/N) tiles (slot s = source rank s); rank r's gathered wire holds all T
// tiles; rank r's flags are N*P words for its mailbox (index s*P + c: source
// s, chunk c) then N*P words for its gathered wire (index N*P + j*P + c: owner
// j, chunk c).
//
// Ordering.  A writer's CTA finishes its stores, meets a CTA barrier, and one
// thread issues a fence and a release store of the call's epoch into the flag;
// a waiter polls the flag with acquire loads until it reaches the epoch, then
// meets a CTA barrier before any thread reads the data (system scope when
// other ranks run on other GPUs, GPU scope when every rank is in the launch).
// The epoch lives in the launching rank's status words: every CTA reads the
// previous call's epoch when it starts and the last CTA to finish stores the
// new one, so a call captured in a CUDA graph advances it on every replay.
// Epochs grow by one per call, so no flag needs resetting; a buffer is never
// rewritten before every reader of the previous call is done with it (a rank
// enters call k+1 only after it has decoded every shard of call k, and every
// shard of call k was reduced only after its mailbox chunks had been read).
//
// Waits are bounded: a wait that sees no progress for timeout_ns (or after
// timeout_ns / 128 polls) records the failure in the caller's status words
// and its CTA stops (the decision is taken at a CTA barrier, so all its
// threads stop together); every other wait of the launch then sees the status
// and stops as well, so a missing rank ends the call with an error instead of
// a hang.  Inside one launch every CTA finishes its phase-A work before its
// first wait and phase-B waits depend only on phase A, phase-C waits only on
// phase B; the launch is cooperative, so all its CTAs are resident together.
//
// One launch may run several ranks (ranks [rank0, rank0 + R)); with R = N it
// is the whole all-reduce in one GPU's memory, the form the tests run.  Ranks
// outside the launch must be another GPU's (or mapped host) memory: two
// launches on one GPU that wait on each other have no guarantee of running at
// the same time, so the C ABI refuses that case.
#include "lpar.h"
#include "lpar_codec.cuh"
#include "lpar_tiles.cuh"

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

namespace lpar {

namespace {

struct PeerPtrs {
    const uint8_t *in[kMaxRanks];      // BF16 inputs (ranks of the launch)
    uint8_t *out[kMaxRanks];           // BF16 outputs (ranks of the launch)
    uint8_t *mbox[kMaxRanks];          // every rank's mailbox
    uint8_t *gath[kMaxRanks];          // every rank's gathered wire
    uint32_t *flags[kMaxRanks];        // every rank's flag words
};

struct PeerGeom {
    unsigned long long T;              // tiles per rank
    unsigned long long slot;           // tiles per mailbox slot: ceil(T / N)
    unsigned long long timeout_ns;
    unsigned P;                        // chunks per shard
    int rank0, R;                      // the ranks this launch runs
    int sys;                           // 1: other ranks run elsewhere (system-scope ordering)
};

// Status words (LPAR_PEER_STATUS_WORDS, in the launching GPU's memory).
constexpr int kStFail = 0, kStPhase = 1, kStRank = 2, kStIndex = 3, kStEpoch = 4, kStDone = 5;

// Chunks per shard.  Every flag costs a CTA barrier, a fence and a wait, so a
// chunk should carry several tiles; a small message should still give every
// CTA work.  Chunk size: about N*T/592 tiles (with every rank in one launch
// that makes about 592 phase-A items, four CTAs on each of 148 SMs), at least
// one and at most kPeerChunkTiles, a whole number of 4-tile groups above four;
// at most kPeerMaxChunks chunks per shard.  Measured on B200 with every rank
// in one launch: 20-30% faster than 16-tile chunks at 1 MiB per rank; from
// 16 MiB it gives 16-tile chunks.  It depends on (N, T) alone, so every rank
// derives the same chunks.
constexpr unsigned kPeerMaxChunks = 1024;
constexpr unsigned kPeerChunkTiles = 16;

inline unsigned peer_chunks(int N, size_t T) {
    const size_t s = (T + (size_t)N - 1) / (size_t)N;
    size_t ct = std::min<size_t>(std::max<size_t>(((size_t)N * T + 591) / 592, 1), kPeerChunkTiles);
    if (ct > 4) ct = (ct + 3) / 4 * 4;
    const size_t c = (s + ct - 1) / ct;
    return (unsigned)std::min<size_t>(std::max<size_t>(c, 1), kPeerMaxChunks);
}

// Flag accesses at the scope of the threads that take part: the whole system
// when other ranks run on other GPUs, this GPU when every rank runs in this
// launch (measured on B200: the system-scope fence makes the all-ranks launch
// 3-4x slower at 16 MiB per rank, and buys nothing there).
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p, int sys) {
    uint32_t v;
    if (sys) asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    else asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v, int sys) {
    if (sys) asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
    else asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence(int sys) {
    if (sys) __threadfence_system();
    else __threadfence();
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t ld_status(const uint32_t *status) {
    return *reinterpret_cast<const volatile uint32_t *>(status);
}

// Chunk c of shard j: tiles [lo, hi); `base` = the shard's first tile.
__device__ __forceinline__ void chunk_tiles(int j, unsigned c, int N, const PeerGeom &g, size_t &lo, size_t &hi,
                                            size_t &base) {
    base = (size_t)j * g.T / (size_t)N;
    const size_t S = (size_t)(j + 1) * g.T / (size_t)N - base;
    lo = base + (size_t)c * S / g.P;
    hi = base + (size_t)(c + 1) * S / g.P;
}

// One thread waits until *flag has reached the epoch.  False when the wait
// gave up (recorded in the status words: fail = 1, the phase, the waiting
// rank, the flag's index) or another wait already had.
__device__ bool wait_flag(const uint32_t *flag, uint32_t epoch, const PeerGeom &g, uint32_t *status, uint32_t phase,
                          int rank, uint32_t index) {
    const unsigned long long t0 = globaltimer_ns();
    const unsigned long long polls = g.timeout_ns / 128 + 1024;
    for (unsigned long long k = 0; k < polls; ++k) {
        if ((int32_t)(ld_acquire(flag, g.sys) - epoch) >= 0) return true;
        if (ld_status(status) != 0) return false;
        if (globaltimer_ns() - t0 > g.timeout_ns) break;
        __nanosleep(200);
    }
    if (atomicCAS(status + kStFail, 0u, 1u) == 0u) {
        status[kStPhase] = phase;
        status[kStRank] = (uint32_t)rank;
        status[kStIndex] = index;
        __threadfence();
    }
    return false;
}

// Every CTA on every way out: the last one to finish (so every CTA has read
// the old epoch) stores the call's epoch for the next call.
__device__ __forceinline__ void finish(uint32_t *status, uint32_t epoch) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(status + kStDone, 1u) == gridDim.x - 1) {
            status[kStDone] = 0;
            *reinterpret_cast<volatile uint32_t *>(status + kStEpoch) = epoch;
            __threadfence();
        }
    }
}

// After the CTA's stores: one thread publishes them with `count` flags
// (flag k at base[k] + index).
__device__ __forceinline__ void publish(uint32_t *const *flag_bases, int count, int first, size_t index,
                                        uint32_t epoch, int sys) {
    __syncthreads();
    if (threadIdx.x == 0) {
        fence(sys);
        for (int q = 0; q < count; ++q) {
            const int r = (first + q) % count;
            st_release(flag_bases[r] + index, epoch, sys);
        }
    }
}

// Coalesced 16-B copy of `bytes` (a multiple of 16) by the whole CTA.
__device__ __forceinline__ void copy16(uint8_t *dst, const uint8_t *src, size_t bytes) {
    for (size_t o = 16u * threadIdx.x; o < bytes; o += 16u * kThreads)
        *reinterpret_cast<uint4 *>(dst + o) = *reinterpret_cast<const uint4 *>(src + o);
}

// Stage 2 of block b of local tile `tile` from N wires (slot bases wp) into
// dst_tile: the arithmetic of reduce_block, with the requantised block stored
// to a tile of the CTA's staging buffer instead of the gathered wire.
template <int C, int N>
__device__ __forceinline__ void peer_reduce_block(const uint8_t *const *wp, size_t tile, int b, uint8_t *dst_tile) {
    Packed<C> q[N];
#pragma unroll
    for (int s = 0; s < N; ++s) load_block(wp[s] + tile * Layout<C>::kTileBytes, b, q[s]);
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.0f;                   // +0.0f, then ranks in ascending order
#pragma unroll
    for (int s = 0; s < N; ++s) accumulate<C>(q[s], acc);
    const float a = absmax_f32x32(acc);
    Packed<C> gb;
    if constexpr (C == kFP8) {
        encode_fp8<false>(acc, a, gb, NoSink{});
    } else if constexpr (C == kMXFP4) {
        encode_mxfp4<false>(acc, a, gb, NoSink{});
    } else {
        const IntScale k = int_scale<Layout<C>::kBits>(a);
        gb.scale = k.bits;
        bool ok = k.fast;
        if constexpr (C == kINT4) {
            if (ok) ok = int4_fast<true, false>(acc, k, gb.w, NoSink{});
        } else {
            if (ok) ok = int3_fast<true, false>(acc, k, gb.q2w, gb.q1w, NoSink{});
        }
        if (!ok) reduce_block_exact<C, false>(wp, N, tile, b, &gb, NoSink{});
    }
    store_block(dst_tile, b, gb);
}

// Phase A: items (chunk c, owner j, rank r), c-major, so the first chunks of
// every shard are published first.
template <int C, int N>
__device__ void peer_phase_a(const PeerPtrs &p, const PeerGeom &g, uint32_t epoch,
                             uint8_t (*stage)[C == kBF16 ? 16 : kStageBytes], uint8_t *wst) {
    constexpr size_t TB = Layout<C>::kTileBytes;
    const int t = threadIdx.x;
    const size_t per_c = (size_t)N * g.R;
    const size_t items = (size_t)g.P * per_c;
    for (size_t i = blockIdx.x; i < items; i += gridDim.x) {
        const unsigned c = (unsigned)(i / per_c);
        const int rem = (int)(i % per_c), j = rem / g.R, r = g.rank0 + rem % g.R;
        size_t lo, hi, base;
        chunk_tiles(j, c, N, g, lo, hi, base);
        if (lo == hi) continue;
        const uint8_t *src = p.in[r] + lo * (kTileElems * 2);
        uint8_t *dst = p.mbox[j] + ((size_t)r * g.slot + (lo - base)) * TB;
        if constexpr (C == kBF16) {
            copy16(dst, src, (hi - lo) * TB);
        } else {
            const size_t groups = (hi - lo + kTilesPerCta - 1) / kTilesPerCta;
            stage_load_chunk(stage[0], src, (int)min((size_t)kTilesPerCta, hi - lo));
            cp_async_commit();
            int buf = 0;
            for (size_t k = 0; k < groups; ++k) {
                const size_t t0 = lo + k * kTilesPerCta;
                const int ntl = (int)min((size_t)kTilesPerCta, hi - t0);
                if (k + 1 < groups)
                    stage_load_chunk(stage[buf ^ 1], src + (k + 1) * (kTilesPerCta * kTileElems * 2),
                                     (int)min((size_t)kTilesPerCta, hi - t0 - kTilesPerCta));
                cp_async_commit();
                cp_async_wait_prev();                            // this group's BF16 has landed
                __syncthreads();                                 // ... for every thread; wst is free
                if (t < ntl * kBlocksPerTile) {
                    uint32_t x16[16];
                    stage_read(stage[buf], t, x16);
                    float x[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) { x[2 * e] = bf16lo(x16[e]); x[2 * e + 1] = bf16hi(x16[e]); }
                    const float a = absmax_bf16x32(x16);
                    Packed<C> q;
                    encode<C, false, false>(x, a, q, NoSink{});
                    // to another GPU: staged, then whole 16-B stores; in this GPU's memory: direct
                    // (measured 2-5% faster with every rank in the launch)
                    if (g.sys) store_block(wst + (t / kBlocksPerTile) * TB, t % kBlocksPerTile, q);
                    else store_block(dst + (k * kTilesPerCta + t / kBlocksPerTile) * TB, t % kBlocksPerTile, q);
                }
                __syncthreads();                                 // wst filled; stage[buf] read by all
                if (g.sys) copy16(dst + k * (kTilesPerCta * TB), wst, (size_t)ntl * TB);
                buf ^= 1;
            }
        }
        publish(p.flags + j, 1, 0, (size_t)r * g.P + c, epoch, g.sys);
    }
}

// Phase B: items (chunk c, owner j) for the launch's ranks j.
template <int C, int N>
__device__ bool peer_phase_b(const PeerPtrs &p, const PeerGeom &g, uint32_t epoch, uint8_t *wst, uint32_t *status) {
    constexpr size_t TB = Layout<C>::kTileBytes;
    const int t = threadIdx.x;
    const size_t items = (size_t)g.P * g.R;
    for (size_t i = blockIdx.x; i < items; i += gridDim.x) {
        const unsigned c = (unsigned)(i / g.R);
        const int j = g.rank0 + (int)(i % g.R);
        size_t lo, hi, base;
        chunk_tiles(j, c, N, g, lo, hi, base);
        if (lo == hi) continue;
        const bool gave_up =
            t < N && !wait_flag(p.flags[j] + (size_t)t * g.P + c, epoch, g, status, 1, j, (uint32_t)(t * g.P + c));
        if (__syncthreads_or(gave_up)) return false;             // else the N chunks are visible to every thread
        const uint8_t *wp[N];
#pragma unroll
        for (int s = 0; s < N; ++s) wp[s] = p.mbox[j] + (size_t)s * g.slot * TB;
        if constexpr (C == kBF16) {
            const size_t nv = (hi - lo) * (TB / 16), l0 = (lo - base) * TB;
            for (size_t v = t; v < nv; v += kThreads) {
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
                for (int s = 0; s < N; ++s) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(wp[s] + l0 + 16 * v);
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[2 * e] = __fadd_rn(acc[2 * e], bf16lo(w[e]));
                        acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], bf16hi(w[e]));
                    }
                }
                const uint4 o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                           pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
#pragma unroll
                for (int q = 0; q < N; ++q)
                    *reinterpret_cast<uint4 *>(p.gath[(j + 1 + q) % N] + lo * TB + 16 * v) = o;
            }
        } else {
            for (size_t t0 = lo; t0 < hi; t0 += kTilesPerCta) {
                const int ntl = (int)min((size_t)kTilesPerCta, hi - t0);
                __syncthreads();                                 // wst is free
                if (t < ntl * kBlocksPerTile)
                    peer_reduce_block<C, N>(wp, (t0 - base) + t / kBlocksPerTile, t % kBlocksPerTile,
                                            wst + (t / kBlocksPerTile) * TB);
                __syncthreads();
#pragma unroll 1
                for (int q = 0; q < N; ++q)                      // every rank, starting after the owner
                    copy16(p.gath[(j + 1 + q) % N] + t0 * TB, wst, (size_t)ntl * TB);
            }
        }
        publish(p.flags, N, j + 1, (size_t)(N + j) * g.P + c, epoch, g.sys);
    }
    return true;
}

// Phase C: items (chunk c, owner j, rank r).
template <int C, int N>
__device__ void peer_phase_c(const PeerPtrs &p, const PeerGeom &g, uint32_t epoch, uint8_t *stage, uint32_t *status) {
    constexpr size_t TB = Layout<C>::kTileBytes;
    const int t = threadIdx.x;
    const size_t per_c = (size_t)N * g.R;
    const size_t items = (size_t)g.P * per_c;
    for (size_t i = blockIdx.x; i < items; i += gridDim.x) {
        const unsigned c = (unsigned)(i / per_c);
        const int rem = (int)(i % per_c), j = rem / g.R, r = g.rank0 + rem % g.R;
        size_t lo, hi, base;
        chunk_tiles(j, c, N, g, lo, hi, base);
        if (lo == hi) continue;
        const size_t fi = (size_t)(N + j) * g.P + c;
        const bool gave_up = t == 0 && !wait_flag(p.flags[r] + fi, epoch, g, status, 2, r, (uint32_t)fi);
        if (__syncthreads_or(gave_up)) return;
        const uint8_t *src = p.gath[r];
        uint8_t *dst = p.out[r];
        if constexpr (C == kBF16) {
            copy16(dst + lo * TB, src + lo * TB, (hi - lo) * TB);
        } else {
            for (size_t t0 = lo; t0 < hi; t0 += kTilesPerCta) {
                const int ntl = (int)min((size_t)kTilesPerCta, hi - t0);
                __syncthreads();                                 // the stage is free
                if (t < ntl * kBlocksPerTile) {
                    Packed<C> q;
                    load_block(src + (t0 + t / kBlocksPerTile) * TB, t % kBlocksPerTile, q);
                    uint32_t o[16];
                    decode<C>(q, o);
                    stage_write(stage, t, o);
                }
                __syncthreads();
#pragma unroll
                for (int k = 0; k < kTilesPerCta; ++k) {
                    const int gi = t + kThreads * k;             // 16-B piece of the group
                    if (gi < ntl * 256)
                        *reinterpret_cast<uint4 *>(dst + t0 * (kTileElems * 2) + 16 * (size_t)gi) =
                            *reinterpret_cast<const uint4 *>(stage + swz(gi >> 2, gi & 3));
                }
            }
        }
    }
}

// Four CTAs per SM (at most 64 registers a thread): measured on B200 with every
// rank in one launch, 10-20% faster than the two or three CTAs per SM the
// unbounded register counts allow, for every codec from 64 MiB per rank on.
template <int C, int N>
__global__ void __launch_bounds__(kThreads, 4) k_allreduce_peer(const __grid_constant__ PeerPtrs p,
                                                             const __grid_constant__ PeerGeom g, uint32_t *status) {
    __shared__ __align__(128) uint8_t stage[2][C == kBF16 ? 16 : kStageBytes];
    __shared__ __align__(16) uint8_t wst[C == kBF16 ? 16 : kTilesPerCta * Layout<C>::kTileBytes];
    __shared__ uint32_t s_epoch;
    if (threadIdx.x == 0) s_epoch = ld_status(status + kStEpoch) + 1u;
    // a failed earlier call: do nothing
    const bool failed = __syncthreads_or(threadIdx.x == 0 && ld_status(status + kStFail) != 0);
    const uint32_t epoch = s_epoch;
    if (!failed) {
        peer_phase_a<C, N>(p, g, epoch, stage, wst);
        if constexpr (C != kBF16) cp_async_wait_all_groups();
        if (peer_phase_b<C, N>(p, g, epoch, wst, status)) peer_phase_c<C, N>(p, g, epoch, stage[0], status);
    }
    finish(status, epoch);
}

template <int C, int N>
lpar_status_t launch_peer_cn(const PeerPtrs &p, const PeerGeom &g, uint32_t *status, cudaStream_t st) {
    const unsigned res = resident_ctas<k_allreduce_peer<C, N>>();
    if (!res) return LPAR_ERR_CUDA;
    const size_t items = (size_t)g.P * N * g.R;
    const unsigned grid = (unsigned)std::min<size_t>(res, items);
    void *args[] = {const_cast<PeerPtrs *>(&p), const_cast<PeerGeom *>(&g), &status};
    if (cudaLaunchCooperativeKernel((const void *)k_allreduce_peer<C, N>, dim3(grid), dim3(kThreads), args, 0, st) ==
        cudaSuccess)
        return LPAR_OK;
    cudaGetLastError();                    // a refused launch leaves no error for later calls to find
    return LPAR_ERR_CUDA;
}

template <int C>
lpar_status_t launch_peer_c(int N, const PeerPtrs &p, const PeerGeom &g, uint32_t *status, cudaStream_t st) {
    switch (N) {
        case 1: return launch_peer_cn<C, 1>(p, g, status, st);
        case 2: return launch_peer_cn<C, 2>(p, g, status, st);
        case 3: return launch_peer_cn<C, 3>(p, g, status, st);
        case 4: return launch_peer_cn<C, 4>(p, g, status, st);
        case 5: return launch_peer_cn<C, 5>(p, g, status, st);
        case 6: return launch_peer_cn<C, 6>(p, g, status, st);
        case 7: return launch_peer_cn<C, 7>(p, g, status, st);
        default: return launch_peer_cn<C, 8>(p, g, status, st);
    }
}

// A buffer of a rank outside the launch must be memory this GPU can reach and
// that another launch (on another GPU) or the host can own: another device's
// memory (peer or IPC-mapped) or mapped host memory.  Memory of the current
// device would mean a second launch on this GPU waiting on this one;
// unregistered host memory is not reachable from the kernel.
bool reachable_elsewhere(const void *ptr, int dev) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeHost) return true;
    return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device != dev;
}

size_t tiles_of(size_t n) { return n / kTileElems; }

}  // namespace
}  // namespace lpar

using namespace lpar;

LPAR_API size_t lpar_peer_mailbox_bytes(int N, size_t n, lpar_codec_t codec) {
    if (N < 1 || N > kMaxRanks || !codec_ok(codec) || n % kTileElems || tiles_of(n) > kMaxTiles) return 0;
    const size_t T = tiles_of(n);
    return (size_t)N * ((T + N - 1) / N) * lpar_tile_bytes(codec);
}

LPAR_API size_t lpar_peer_gather_bytes(size_t n, lpar_codec_t codec) {
    if (!codec_ok(codec) || n % kTileElems || tiles_of(n) > kMaxTiles) return 0;
    return tiles_of(n) * lpar_tile_bytes(codec);
}

LPAR_API size_t lpar_peer_flag_bytes(int N, size_t n) {
    if (N < 1 || N > kMaxRanks || n % kTileElems || tiles_of(n) > kMaxTiles) return 0;
    if (n == 0) return 0;
    return 2 * (size_t)N * peer_chunks(N, tiles_of(n)) * sizeof(uint32_t);
}

LPAR_API lpar_status_t lpar_allreduce_peer(
    const void *const *inputs, void *const *outputs, void *const *mailboxes, void *const *gathered,
    void *const *flags, int N, int rank0, int ranks, size_t n, lpar_codec_t codec, uint64_t timeout_ns,
    uint32_t *status, cudaStream_t stream) {
    if (N < 1 || N > kMaxRanks || rank0 < 0 || ranks < 1 || rank0 + ranks > N) return LPAR_ERR_INVALID_ARG;
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    if (n % kTileElems || tiles_of(n) > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (!inputs || !outputs || !mailboxes || !gathered || !flags || !status || timeout_ns == 0)
        return LPAR_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(status) & 15u) return LPAR_ERR_MISALIGNED;
    PeerPtrs p{};
    for (int r = 0; r < N; ++r) {
        if (!mailboxes[r] || !gathered[r] || !flags[r]) return LPAR_ERR_INVALID_ARG;
        if (!aligned16(mailboxes[r]) || !aligned16(gathered[r]) || !aligned16(flags[r])) return LPAR_ERR_MISALIGNED;
        p.mbox[r] = static_cast<uint8_t *>(mailboxes[r]);
        p.gath[r] = static_cast<uint8_t *>(gathered[r]);
        p.flags[r] = static_cast<uint32_t *>(flags[r]);
        if (r >= rank0 && r < rank0 + ranks) {
            if (!inputs[r] || !outputs[r]) return LPAR_ERR_INVALID_ARG;
            if (!aligned16(inputs[r]) || !aligned16(outputs[r])) return LPAR_ERR_MISALIGNED;
            p.in[r] = static_cast<const uint8_t *>(inputs[r]);
            p.out[r] = static_cast<uint8_t *>(outputs[r]);
        }
    }
    if (n == 0) return LPAR_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LPAR_ERR_CUDA;
    if (ranks < N) {
        for (int r = 0; r < N; ++r) {
            if (r >= rank0 && r < rank0 + ranks) continue;
            if (!reachable_elsewhere(mailboxes[r], dev) || !reachable_elsewhere(gathered[r], dev) ||
                !reachable_elsewhere(flags[r], dev))
                return LPAR_ERR_INVALID_ARG;
        }
    }
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) return LPAR_ERR_CUDA;
    if (!coop) return LPAR_ERR_UNSUPPORTED;
    const size_t T = tiles_of(n);
    PeerGeom g{};
    g.T = T;
    g.slot = (T + N - 1) / N;
    g.timeout_ns = timeout_ns;
    g.P = peer_chunks(N, T);
    g.rank0 = rank0;
    g.R = ranks;
    g.sys = ranks < N;
    NvtxRange nvtx("lpar_allreduce_peer");
    switch (codec) {
        case LPAR_CODEC_BF16: return launch_peer_c<kBF16>(N, p, g, status, stream);
        case LPAR_CODEC_FP8_E4M3: return launch_peer_c<kFP8>(N, p, g, status, stream);
        case LPAR_CODEC_INT4: return launch_peer_c<kINT4>(N, p, g, status, stream);
        case LPAR_CODEC_INT3: return launch_peer_c<kINT3>(N, p, g, status, stream);
        default: return launch_peer_c<kMXFP4>(N, p, g, status, stream);
    }
}

// ---- buffers shared between processes (CUDA IPC) ---------------------------------
LPAR_API lpar_status_t lpar_peer_alloc(size_t bytes, void **ptr) {
    if (!ptr || bytes == 0) return LPAR_ERR_INVALID_ARG;
    *ptr = nullptr;
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
        cudaGetLastError();
        return LPAR_ERR_CUDA;
    }
    if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(p);
        return LPAR_ERR_CUDA;
    }
    *ptr = p;
    return LPAR_OK;
}

LPAR_API lpar_status_t lpar_peer_free(void *ptr) {
    if (!ptr) return LPAR_ERR_INVALID_ARG;
    return cudaFree(ptr) == cudaSuccess ? LPAR_OK : LPAR_ERR_CUDA;
}

LPAR_API lpar_status_t lpar_peer_export(const void *ptr, unsigned char *handle) {
    if (!ptr || !handle) return LPAR_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, const_cast<void *>(ptr)) != cudaSuccess) {
        cudaGetLastError();
        return LPAR_ERR_CUDA;
    }
    static_assert(sizeof(h) == LPAR_PEER_HANDLE_BYTES, "IPC handle size");
    std::copy(reinterpret_cast<const unsigned char *>(&h), reinterpret_cast<const unsigned char *>(&h) + sizeof(h),
              handle);
    return LPAR_OK;
}

LPAR_API lpar_status_t lpar_peer_import(const unsigned char *handle, void **ptr) {
    if (!handle || !ptr) return LPAR_ERR_INVALID_ARG;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::copy(handle, handle + sizeof(h), reinterpret_cast<unsigned char *>(&h));
    void *p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return LPAR_ERR_CUDA;
    }
    *ptr = p;
    return LPAR_OK;
}

LPAR_API lpar_status_t lpar_peer_close(void *ptr) {
    if (!ptr) return LPAR_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(ptr) == cudaSuccess ? LPAR_OK : LPAR_ERR_CUDA;
}

