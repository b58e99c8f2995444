// lpar_kernels.cu -- sm_100a kernels of the compressed all-reduce and the C ABI.
//
// Stages (two-shot all-reduce, "RCCLX: Innovating GPU communications on AMD
// platforms", Direct Data Access: reduce-scatter then all-gather; FP32
// compute per its Low-Precision Collectives section; tile formats per
// "QuickReduce INT3 Quantization and Benchmarking on MI355", Summary/Method):
//   K1  k_quantize      BF16 -> wire, all N ranks in one persistent launch
//   K2  k_reduce<.., false>  N wires -> FP32 sum in rank order -> requantised
//                        gathered wire
//   K23 k_reduce<.., true>   K2 plus the decode of the gathered block straight
//                        from registers into every rank's BF16 output
//   K3  k_decode        gathered wire -> BF16 into every rank's output
//   K123 all three stages in one kernel (the default schedule), in three
//        forms: k_allreduce_tile (one tile per CTA, the ranks' stage 1 spread
//        over the CTA's threads: small messages), and the persistent
//        k_allreduce_single_warp (warp-local, no CTA barrier) and
//        k_allreduce_single (CTA-wide, output by bulk copies from 128 MiB of
//        input); launch_single_cn picks one by codec, N and size
// The BF16 passthrough uses k_bf16_reduce (FP32 sum, one BF16 rounding) and
// k_broadcast (plain copies).  The one-shot schedule's kernel lives with the
// standalone collectives (lpar_collectives.cu), the binary32 all-reduce in
// lpar_f32.cu.  The work decomposition and the staging are described in
// lpar_tiles.cuh.
#include "lpar.h"
#include "lpar_codec.cuh"
#include "lpar_tiles.cuh"

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace lpar {

// ---------------------------------------------------------------------------
// K1: stage 1 for every rank.  Persistent: CTA b handles the work items
// (chunk c, rank r) for c = b, b + gridDim.x, ... and r = 0..N-1 (a chunk is 4
// tiles).  The BF16 chunk of the next item is copied into the other half of a
// double-buffered stage (cp.async) while the current one is encoded.
// ---------------------------------------------------------------------------
template <int C>
__global__ void __launch_bounds__(kThreads, 5) k_quantize(const __grid_constant__ InPtrs in,
                                                       const __grid_constant__ OutPtrs wire, size_t tiles,
                                                       unsigned chunks, int N) {
    __shared__ __align__(128) uint8_t stage[2][kStageBytes];
    const int t = threadIdx.x;
    // work item = (chunk c, rank r); a CTA walks r = 0..N-1, then c += gridDim.x
    unsigned c = blockIdx.x;
    int r = 0;
    if (c < chunks) {
        const size_t tile0 = (size_t)c * kTilesPerCta;
        stage_load_chunk(stage[0], in.p[0] + tile0 * (kTileElems * 2), (int)min((size_t)kTilesPerCta, tiles - tile0));
    }
    cp_async_commit();
    int buf = 0;
    while (c < chunks) {
        unsigned cn = c;
        int rn = r + 1;
        if (rn == N) { rn = 0; cn += gridDim.x; }
        if (cn < chunks) {
            const size_t tn = (size_t)cn * kTilesPerCta;
            stage_load_chunk(stage[buf ^ 1], in.p[rn] + tn * (kTileElems * 2),
                             (int)min((size_t)kTilesPerCta, tiles - tn));
        }
        cp_async_commit();
        cp_async_wait_prev();                          // this item's copies have landed
        __syncthreads();
        const size_t tile0 = (size_t)c * kTilesPerCta;
        const int ntiles = (int)min((size_t)kTilesPerCta, tiles - tile0);
        if (t < ntiles * kBlocksPerTile) {
            uint32_t x16[16];
            stage_read(stage[buf], t, x16);
            float x[32];
#pragma unroll
            for (int k = 0; k < 16; ++k) { x[2 * k] = bf16lo(x16[k]); x[2 * k + 1] = bf16hi(x16[k]); }
            const float a = absmax_bf16x32(x16);
            Packed<C> p;
            encode<C, false, false>(x, a, p, NoSink{});
            store_block(wire.p[r] + (tile0 + t / kBlocksPerTile) * Layout<C>::kTileBytes, t % kBlocksPerTile, p);
        }
        __syncthreads();                               // stage[buf] is refilled next iteration
        buf ^= 1;
        c = cn;
        r = rn;
    }
}

// ---------------------------------------------------------------------------
// K2 / K23: tiles [tile_begin, tile_end) of N wires -> gathered wire (and,
// when FUSED, the decoded BF16 result into every out[r]).
// ---------------------------------------------------------------------------
template <int C, int N, bool FUSED>
__global__ void __launch_bounds__(kThreads) k_reduce(const __grid_constant__ InPtrs wires, uint8_t *gather,
                                                     const __grid_constant__ OutPtrs out, size_t tile_begin,
                                                     size_t tile_end) {
    __shared__ __align__(128) uint8_t stage[FUSED ? kStageBytes : 16];
    const int t = threadIdx.x;
    const size_t tile0 = tile_begin + (size_t)blockIdx.x * kTilesPerCta;
    const int ntiles = (int)min((size_t)kTilesPerCta, tile_end - tile0);
    if (t < ntiles * kBlocksPerTile) {
        const size_t tile = tile0 + t / kBlocksPerTile;
        const int b = t % kBlocksPerTile;
        if constexpr (FUSED) reduce_block<C, N, true>(wires.p, tile, b, gather, StageSink{stage, t});
        else reduce_block<C, N, false>(wires.p, tile, b, gather, NoSink{});
    }
    if (FUSED) {
        __syncthreads();
        stage_to_outputs(stage, out, N, tile0 * (kTileElems * 2), ntiles);
    }
}

// ---------------------------------------------------------------------------
// K123 (single-pass schedule): one persistent kernel.  For each chunk of 4
// tiles a CTA quantises the chunk of every rank into that rank's wire (stage
// 1), then reduces the chunk from the wires it has just written, requantises
// it into the gathered wire and decodes it into every rank's output (stages 2
// and 3).  A tile's result depends only on the same tile of every rank, so no
// CTA waits for another; each thread reads back only wire blocks it wrote
// itself (same thread, program order).  The next rank's BF16 chunk is
// prefetched with cp.async while the current one is processed.
// ---------------------------------------------------------------------------
// Output of the single-pass kernel.  BULK: the decoded chunk is staged in
// element order and sent by the TMA engine (bulk shared->global copies), so a
// CTA moves on while the copies drain; otherwise every thread stores its
// share of the staged chunk to each output.  The copies add about 2 us of
// latency to a call and win on throughput, so the launcher takes them from
// kBulkMinBytes of input (N x message bytes) on (measured on B200 with the
// variants timed alternately in one process: below about 128 MiB the
// synchronous stores are faster, above it the copies by 2-12%).
constexpr size_t kBulkMinBytes = (size_t)128 << 20;

// Stages in the single-pass ring (measured the same way): with the bulk
// copies, four -- three CTAs per SM, 80 registers a thread -- for FP8 and,
// from four ranks on, for INT4 and MXFP4; three -- four CTAs per SM, 64
// registers -- for INT3 (its ALU-bound encode wants the warps) and for INT4
// and MXFP4 with fewer ranks.  The synchronous stores need three.
template <int C, int N, bool BULK>
__host__ __device__ constexpr int ring_stages() {
    return (BULK && (C == kFP8 || (C != kINT3 && N >= 4))) ? 4 : 3;
}
template <int C, int N, bool BULK>
__host__ __device__ constexpr int ring_smem() { return ring_stages<C, N, BULK>() * kStageBytes; }

template <int C, int N, bool BULK>
__global__ void __launch_bounds__(kThreads, ring_stages<C, N, BULK>() == 3 ? 4 : 3)
    k_allreduce_single(const __grid_constant__ InPtrs in, const __grid_constant__ OutPtrs wire, uint8_t *gather,
                       const __grid_constant__ OutPtrs out, size_t tiles, unsigned chunks) {
    // A ring of S BF16 stages: item i is staged in stage i % S while item i + 1
    // is prefetched, and stage i % S is refilled S - 1 items later, after a
    // barrier that every thread passes only once done with it -- one barrier
    // per item.  The decoded chunk is staged in place of the last rank's input
    // (each thread writes only the 64-B region it read).  Synchronous output:
    // every thread copies its share to the N outputs before the next item's
    // barrier.  Bulk output: the chunk leaves through copies issued by lanes
    // of warp 0, which wait for them to finish reading before the barrier
    // that precedes the stage's refill -- the next item's (S = 3) or the one
    // after (S = 4), so that with four stages the copies overlap the encode
    // of the next item.
    constexpr int S = ring_stages<C, N, BULK>();
    static_assert(S == 3 || S == 4, "ring of three or four stages");
    extern __shared__ __align__(1024) uint8_t ring[];
    const int t = threadIdx.x;
    unsigned c = blockIdx.x;
    if (c >= chunks) return;
    stage_load_chunk(ring, in.p[0] + (size_t)c * kTilesPerCta * (kTileElems * 2),
                     (int)min((size_t)kTilesPerCta, tiles - (size_t)c * kTilesPerCta));
    cp_async_commit();
    int buf = 0;
    for (; c < chunks; c += gridDim.x) {
        const size_t tile0 = (size_t)c * kTilesPerCta;
        const int ntiles = (int)min((size_t)kTilesPerCta, tiles - tile0);
        const bool active = t < ntiles * kBlocksPerTile;
        const size_t tile = tile0 + t / kBlocksPerTile;
        const int b = t % kBlocksPerTile;
        int last = buf;
#pragma unroll 1
        for (int r = 0; r < N; ++r) {
            // prefetch the next item: rank r+1 of this chunk, or rank 0 of the next chunk
            const int nb = buf + 1 == S ? 0 : buf + 1;
            const unsigned cn = (r + 1 < N) ? c : c + gridDim.x;
            if (cn < chunks) {
                const size_t tn = (size_t)cn * kTilesPerCta;
                stage_load_chunk(ring + nb * kStageBytes, in.p[(r + 1 < N) ? r + 1 : 0] + tn * (kTileElems * 2),
                                 (int)min((size_t)kTilesPerCta, tiles - tn));
            }
            cp_async_commit();
            cp_async_wait_prev();
            if constexpr (BULK) {
                if constexpr (S == 3) {                // the last chunk's copies
                    if (r == 0 && t < 32) bulk_wait_read<0>();
                } else if constexpr (N == 1) {         // the copies of the chunk before last
                    if (t < 32) bulk_wait_read<1>();
                } else {                               // the last chunk's copies, from its second item on
                    if (r == 1 && t < 32) bulk_wait_read<0>();
                }
            }
            __syncthreads();                           // item landed; stage nb's old item is done
            if (active) {
                uint32_t x16[16];
                stage_read(ring + buf * kStageBytes, t, x16);
                float x[32];
#pragma unroll
                for (int k = 0; k < 16; ++k) { x[2 * k] = bf16lo(x16[k]); x[2 * k + 1] = bf16hi(x16[k]); }
                const float a = absmax_bf16x32(x16);
                Packed<C> p;
                encode<C, false, false>(x, a, p, NoSink{});
                store_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
            }
            last = buf;
            buf = nb;
        }
        uint8_t *const so = ring + last * kStageBytes;
        if constexpr (BULK) {
            if (active) reduce_block<C, N, true>(wire.p, tile, b, gather, StageSinkLinear{so, t});
            fence_async_smem();
            __syncthreads();
            if (t < N) bulk_store(out.p[t] + tile0 * (kTileElems * 2), so, (unsigned)ntiles * (kTileElems * 2));
            if (t < 32) bulk_commit();
        } else {
            if (active) reduce_block<C, N, true>(wire.p, tile, b, gather, StageSink{so, t});
            __syncthreads();
            stage_to_outputs(so, out, N, tile0 * (kTileElems * 2), ntiles);
        }
    }
    if constexpr (BULK) {
        if (t < 32) bulk_wait_read<0>();              // the stage outlives no copy that reads it
    }
}

// K123, warp-local form (issue-bound cases: INT3 with few ranks, and the
// smaller messages of INT4 and MXFP4).  Every warp works on its own half tile
// of the chunk (blocks 32w .. 32w+31) and touches only its own 2 KiB of each
// stage: its lanes copy them in, read them, stage the decoded blocks there and
// store them to every output, so warps never wait for each other (__syncwarp
// only).  A ring of three stages per warp: item i is staged in stage i % 3
// while item i + 1 is prefetched, and refilled two items later, after the
// warp's next __syncwarp.  The decoded chunk is staged in place of the last
// rank's input.  Without CTA barriers the warps drift apart, which costs DRAM
// efficiency when HBM is the bound: there the CTA-wide form is faster.
// Three CTAs per SM (24 warps, 80 registers a thread) measured 3.6% faster
// than four (64 registers) for INT3 at two ranks and 1 GiB, equal elsewhere.
template <int C, int N>
__global__ void __launch_bounds__(kThreads, 3)
    k_allreduce_single_warp(const __grid_constant__ InPtrs in, const __grid_constant__ OutPtrs wire, uint8_t *gather,
                            const __grid_constant__ OutPtrs out, size_t tiles, unsigned chunks) {
    constexpr int S = 3;
    extern __shared__ __align__(1024) uint8_t ring[];
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int wt = w >> 1;                                 // the warp's tile within a chunk
    unsigned c = blockIdx.x;
    if (c >= chunks) return;
    auto has = [&](unsigned cc) { return (size_t)cc * kTilesPerCta + wt < tiles; };
    if (has(c)) warp_load(ring, in.p[0] + (size_t)c * kTilesPerCta * (kTileElems * 2), w, lane);
    cp_async_commit();
    int buf = 0;
    for (; c < chunks; c += gridDim.x) {
        const size_t tile0 = (size_t)c * kTilesPerCta;
        const bool active = has(c);
        const size_t tile = tile0 + wt;
        const int b = t % kBlocksPerTile;
        int last = buf;
#pragma unroll 1
        for (int r = 0; r < N; ++r) {
            // prefetch the next item: rank r+1 of this chunk, or rank 0 of the next chunk
            const int nb = buf + 1 == S ? 0 : buf + 1;
            const unsigned cn = (r + 1 < N) ? c : c + gridDim.x;
            if (cn < chunks && has(cn))
                warp_load(ring + nb * kStageBytes,
                          in.p[(r + 1 < N) ? r + 1 : 0] + (size_t)cn * kTilesPerCta * (kTileElems * 2), w, lane);
            cp_async_commit();
            cp_async_wait_prev();
            __syncwarp();                                  // the warp's item landed
            if (active) {
                uint32_t x16[16];
                stage_read(ring + buf * kStageBytes, t, x16);
                float x[32];
#pragma unroll
                for (int k = 0; k < 16; ++k) { x[2 * k] = bf16lo(x16[k]); x[2 * k + 1] = bf16hi(x16[k]); }
                const float a = absmax_bf16x32(x16);
                Packed<C> p;
                encode<C, false, false>(x, a, p, NoSink{});
                store_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
            }
            last = buf;
            buf = nb;
        }
        uint8_t *const so = ring + last * kStageBytes;
        if (active) reduce_block<C, N, true>(wire.p, tile, b, gather, StageSink{so, t});
        __syncwarp();
        if (active) warp_to_outputs(so, out, N, tile0 * (kTileElems * 2), w, lane);
    }
}

// ---------------------------------------------------------------------------
// K123, rank-parallel form for small messages: one tile per CTA, the N ranks'
// stage 1 spread over the CTA's threads.  A small message fills few CTAs of
// the persistent forms, each encoding the N ranks of its chunk one after
// another; here every tile has its own CTA and the N x 64 block encodes of a
// tile run side by side (thread t encodes block t % 64 of rank t / 64, then of
// rank t / 64 + 4), so the call's dependent chain holds one or two encodes
// instead of N.  The CTA copies the N BF16 tiles into shared memory (one
// swizzled 4-KiB region per rank), writes the N stage-1 wire blocks, and after
// one barrier (which makes the CTA's global writes visible to all its threads)
// threads 0..63 read the N wire blocks of their block back, reduce, requantise
// into the gathered wire and decode into rank 0's region, which all threads
// then store to every output with coalesced 16-B stores.
// ---------------------------------------------------------------------------
template <int C, int N>
__global__ void __launch_bounds__(kThreads) k_allreduce_tile(const __grid_constant__ InPtrs in,
                                                             const __grid_constant__ OutPtrs wire, uint8_t *gather,
                                                             const __grid_constant__ OutPtrs out) {
    constexpr int kTileBytesBf16 = kTileElems * 2;               // 4 KiB: 64 blocks of 64 B
    __shared__ __align__(128) uint8_t stage[N * kTileBytesBf16];
    const int t = threadIdx.x;
    const size_t tile = blockIdx.x;
#pragma unroll
    for (int r = 0; r < N; ++r)                                  // piece t of every rank's tile
        cp_async16(stage + r * kTileBytesBf16 + swz(t >> 2, t & 3), in.p[r] + tile * kTileBytesBf16 + 16 * t);
    cp_async_commit();
    cp_async_wait_all_groups();
    __syncthreads();
#pragma unroll
    for (int k = 0; k < (N + 3) / 4; ++k) {                      // stage 1: block b of rank r
        const int idx = t + kThreads * k, r = idx >> 6, b = idx & 63;
        if (r < N) {
            uint32_t x16[16];
            stage_read(stage + r * kTileBytesBf16, b, x16);
            float x[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) { x[2 * j] = bf16lo(x16[j]); x[2 * j + 1] = bf16hi(x16[j]); }
            const float a = absmax_bf16x32(x16);
            Packed<C> p;
            encode<C, false, false>(x, a, p, NoSink{});
            store_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
        }
    }
    __syncthreads();                                             // wire blocks visible; rank 0's region free
    if (t < kBlocksPerTile) reduce_block<C, N, true>(wire.p, tile, t, gather, StageSink{stage, t});
    __syncthreads();
    const uint4 d = *reinterpret_cast<const uint4 *>(stage + swz(t >> 2, t & 3));
#pragma unroll
    for (int r = 0; r < N; ++r) *reinterpret_cast<uint4 *>(out.p[r] + tile * kTileBytesBf16 + 16 * t) = d;
}

// ---------------------------------------------------------------------------
// K3: gathered wire -> BF16 in every out[r].  grid = ceil(tiles / 4).
// ---------------------------------------------------------------------------
template <int C>
__global__ void __launch_bounds__(kThreads) k_decode(const uint8_t *wire, OutPtrs out, int N, size_t tiles) {
    __shared__ __align__(128) uint8_t stage[kStageBytes];
    const int t = threadIdx.x;
    const size_t tile0 = (size_t)blockIdx.x * kTilesPerCta;
    const int ntiles = (int)min((size_t)kTilesPerCta, tiles - tile0);
    if (t < ntiles * kBlocksPerTile) {
        Packed<C> p;
        load_block(wire + (tile0 + t / kBlocksPerTile) * Layout<C>::kTileBytes, t % kBlocksPerTile, p);
        uint32_t o[16];
        decode<C>(p, o);
        stage_write(stage, t, o);
    }
    __syncthreads();
    stage_to_outputs(stage, out, N, tile0 * (kTileElems * 2), ntiles);
}

// ---------------------------------------------------------------------------
// BF16 passthrough: 8 elements (16 B) per thread, all accesses coalesced.
// ---------------------------------------------------------------------------
template <int N, bool FUSED>
__global__ void __launch_bounds__(kThreads) k_bf16_reduce(InPtrs in, uint8_t *gather, OutPtrs out,
                                                          size_t v_begin, size_t v_end) {
    const size_t i = v_begin + (size_t)blockIdx.x * kThreads + threadIdx.x;   // 16-B vector index
    if (i >= v_end) return;
    uint4 x[N];
#pragma unroll
    for (int r = 0; r < N; ++r) x[r] = *reinterpret_cast<const uint4 *>(in.p[r] + 16 * i);
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
    for (int r = 0; r < N; ++r) {
        const uint32_t w[4] = {x[r].x, x[r].y, x[r].z, x[r].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[2 * k] = __fadd_rn(acc[2 * k], bf16lo(w[k]));
            acc[2 * k + 1] = __fadd_rn(acc[2 * k + 1], bf16hi(w[k]));
        }
    }
    const uint4 o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                               pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    *reinterpret_cast<uint4 *>(gather + 16 * i) = o;
    if (FUSED) {
#pragma unroll
        for (int r = 0; r < N; ++r) *reinterpret_cast<uint4 *>(out.p[r] + 16 * i) = o;
    }
}

__global__ void __launch_bounds__(kThreads) k_broadcast(const uint8_t *src, OutPtrs dst, int N, size_t nvec) {
    const size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= nvec) return;
    const uint4 d = *reinterpret_cast<const uint4 *>(src + 16 * i);
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r)
        if (r < N) *reinterpret_cast<uint4 *>(dst.p[r] + 16 * i) = d;
}

// ---------------------------------------------------------------------------
// Host-side launchers (no validation here; the C ABI validates first).
// ---------------------------------------------------------------------------
static inline unsigned grid_for_tiles(size_t tiles) { return (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta); }

template <int C>
static void launch_quantize_c(const InPtrs &in, const OutPtrs &wire, int N, size_t tiles, cudaStream_t st) {
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    const unsigned res = resident_ctas<k_quantize<C>>();
    // every CTA walks all N ranks of its chunks: size the grid in chunks
    const unsigned per_rank = (res ? res : 148u * 4u);
    const unsigned grid = std::min<unsigned>(chunks, std::max<unsigned>(1u, per_rank));
    k_quantize<C><<<grid, kThreads, 0, st>>>(in, wire, tiles, chunks, N);
}

static void launch_quantize(int codec, const InPtrs &in, const OutPtrs &wire, int N, size_t tiles, cudaStream_t st) {
    switch (codec) {
    case kINT4: launch_quantize_c<kINT4>(in, wire, N, tiles, st); break;
    case kINT3: launch_quantize_c<kINT3>(in, wire, N, tiles, st); break;
    case kFP8: launch_quantize_c<kFP8>(in, wire, N, tiles, st); break;
    case kMXFP4: launch_quantize_c<kMXFP4>(in, wire, N, tiles, st); break;
    default: break;
    }
}

template <int C, bool FUSED>
static void launch_reduce_c(const InPtrs &w, int N, uint8_t *g, const OutPtrs &o, size_t t0, size_t t1, cudaStream_t st) {
    const unsigned grid = grid_for_tiles(t1 - t0);
    switch (N) {
    case 1: k_reduce<C, 1, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 2: k_reduce<C, 2, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 3: k_reduce<C, 3, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 4: k_reduce<C, 4, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 5: k_reduce<C, 5, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 6: k_reduce<C, 6, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 7: k_reduce<C, 7, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    case 8: k_reduce<C, 8, FUSED><<<grid, kThreads, 0, st>>>(w, g, o, t0, t1); break;
    default: break;
    }
}

template <bool FUSED>
static void launch_reduce(int codec, const InPtrs &w, int N, uint8_t *g, const OutPtrs &o, size_t t0, size_t t1,
                          cudaStream_t st) {
    switch (codec) {
    case kINT4: launch_reduce_c<kINT4, FUSED>(w, N, g, o, t0, t1, st); break;
    case kINT3: launch_reduce_c<kINT3, FUSED>(w, N, g, o, t0, t1, st); break;
    case kFP8: launch_reduce_c<kFP8, FUSED>(w, N, g, o, t0, t1, st); break;
    case kMXFP4: launch_reduce_c<kMXFP4, FUSED>(w, N, g, o, t0, t1, st); break;
    default: break;
    }
}

template <bool FUSED>
static void launch_bf16_reduce(const InPtrs &in, int N, uint8_t *g, const OutPtrs &o, size_t v0, size_t v1,
                               cudaStream_t st) {
    const unsigned grid = (unsigned)((v1 - v0 + kThreads - 1) / kThreads);
    switch (N) {
    case 1: k_bf16_reduce<1, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 2: k_bf16_reduce<2, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 3: k_bf16_reduce<3, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 4: k_bf16_reduce<4, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 5: k_bf16_reduce<5, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 6: k_bf16_reduce<6, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 7: k_bf16_reduce<7, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    case 8: k_bf16_reduce<8, FUSED><<<grid, kThreads, 0, st>>>(in, g, o, v0, v1); break;
    default: break;
    }
}

template <int C, int N, bool BULK>
static bool launch_single_cnb(const InPtrs &in, const OutPtrs &wire, uint8_t *g, const OutPtrs &o, size_t tiles,
                              cudaStream_t st) {
    constexpr int smem = ring_smem<C, N, BULK>();
    if (!allow_dynamic_smem<k_allreduce_single<C, N, BULK>>(smem)) return false;
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    const unsigned res = resident_ctas<k_allreduce_single<C, N, BULK>>(smem);
    const unsigned grid = std::min<unsigned>(chunks, std::max<unsigned>(1u, res ? res : 148u * 3u));
    k_allreduce_single<C, N, BULK><<<grid, kThreads, smem, st>>>(in, wire, g, o, tiles, chunks);
    return true;
}

template <int C, int N>
static bool launch_single_warp(const InPtrs &in, const OutPtrs &wire, uint8_t *g, const OutPtrs &o, size_t tiles,
                               cudaStream_t st) {
    constexpr int smem = 3 * kStageBytes;
    if (!allow_dynamic_smem<k_allreduce_single_warp<C, N>>(smem)) return false;
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    const unsigned res = resident_ctas<k_allreduce_single_warp<C, N>>(smem);
    const unsigned grid = std::min<unsigned>(chunks, std::max<unsigned>(1u, res ? res : 148u * 4u));
    k_allreduce_single_warp<C, N><<<grid, kThreads, smem, st>>>(in, wire, g, o, tiles, chunks);
    return true;
}

template <int C, int N>
static bool launch_tile(const InPtrs &in, const OutPtrs &wire, uint8_t *g, const OutPtrs &o, size_t tiles,
                        cudaStream_t st) {
    k_allreduce_tile<C, N><<<(unsigned)tiles, kThreads, 0, st>>>(in, wire, g, o);
    return true;
}

// Which form of K123 runs (measured on B200, the forms timed alternately in one
// process): the rank-parallel tile kernel up to kTileFormMaxTiles tiles per
// rank; above that the warp-local kernel for INT3 with one or two ranks at any size
// (7-11% faster: its encode is issue-bound and the CTA barriers cost issue
// slots) and for INT3 below kInt3WarpMaxBytes of input, and for INT4 and MXFP4
// below kBulkMinBytes (up to 11% faster there); the CTA-wide kernel otherwise
// (HBM-bound: 5-15% faster, with the bulk copies from kBulkMinBytes), and
// always for FP8.
constexpr size_t kInt3WarpMaxBytes = (size_t)512 << 20;


template <int C, int N>
static bool launch_single_cn(const InPtrs &in, const OutPtrs &wire, uint8_t *g, const OutPtrs &o, size_t tiles,
                             cudaStream_t st) {
    const size_t in_bytes = (size_t)N * tiles * (kTileElems * 2);
    if (tiles <= kTileFormMaxTiles<C>()) return launch_tile<C, N>(in, wire, g, o, tiles, st);
    if constexpr (C == kFP8) {
        if (in_bytes >= kBulkMinBytes) return launch_single_cnb<C, N, true>(in, wire, g, o, tiles, st);
        return launch_single_cnb<C, N, false>(in, wire, g, o, tiles, st);
    } else {
        const bool warp = C == kINT3 ? (N <= 2 || in_bytes < kInt3WarpMaxBytes) : in_bytes < kBulkMinBytes;
        if (warp) return launch_single_warp<C, N>(in, wire, g, o, tiles, st);
        return launch_single_cnb<C, N, true>(in, wire, g, o, tiles, st);
    }
}

template <int C>
static bool launch_single_c(const InPtrs &in, const OutPtrs &wire, int N, uint8_t *g, const OutPtrs &o,
                            size_t tiles, cudaStream_t st) {
    switch (N) {
    case 1: return launch_single_cn<C, 1>(in, wire, g, o, tiles, st);
    case 2: return launch_single_cn<C, 2>(in, wire, g, o, tiles, st);
    case 3: return launch_single_cn<C, 3>(in, wire, g, o, tiles, st);
    case 4: return launch_single_cn<C, 4>(in, wire, g, o, tiles, st);
    case 5: return launch_single_cn<C, 5>(in, wire, g, o, tiles, st);
    case 6: return launch_single_cn<C, 6>(in, wire, g, o, tiles, st);
    case 7: return launch_single_cn<C, 7>(in, wire, g, o, tiles, st);
    case 8: return launch_single_cn<C, 8>(in, wire, g, o, tiles, st);
    default: return false;
    }
}

static bool launch_single(int codec, const InPtrs &in, const OutPtrs &wire, int N, uint8_t *g, const OutPtrs &o,
                          size_t tiles, cudaStream_t st) {
    switch (codec) {
    case kINT4: return launch_single_c<kINT4>(in, wire, N, g, o, tiles, st);
    case kINT3: return launch_single_c<kINT3>(in, wire, N, g, o, tiles, st);
    case kFP8: return launch_single_c<kFP8>(in, wire, N, g, o, tiles, st);
    case kMXFP4: return launch_single_c<kMXFP4>(in, wire, N, g, o, tiles, st);
    default: return false;
    }
}

static void launch_decode(int codec, const uint8_t *wire, const OutPtrs &o, int N, size_t tiles, cudaStream_t st) {
    const unsigned grid = grid_for_tiles(tiles);
    switch (codec) {
    case kINT4: k_decode<kINT4><<<grid, kThreads, 0, st>>>(wire, o, N, tiles); break;
    case kINT3: k_decode<kINT3><<<grid, kThreads, 0, st>>>(wire, o, N, tiles); break;
    case kFP8: k_decode<kFP8><<<grid, kThreads, 0, st>>>(wire, o, N, tiles); break;
    case kMXFP4: k_decode<kMXFP4><<<grid, kThreads, 0, st>>>(wire, o, N, tiles); break;
    default: break;
    }
}

static void launch_broadcast(const uint8_t *src, const OutPtrs &o, int N, size_t bytes, cudaStream_t st) {
    const size_t nvec = bytes / 16;
    const unsigned grid = (unsigned)((nvec + kThreads - 1) / kThreads);
    k_broadcast<<<grid, kThreads, 0, st>>>(src, o, N, nvec);
}

}  // namespace lpar

using namespace lpar;

// ---------------------------------------------------------------------------
// The C ABI (validation first, then the launches).
// ---------------------------------------------------------------------------
LPAR_API size_t lpar_tile_bytes(lpar_codec_t codec) {
    switch (codec) {
    case LPAR_CODEC_BF16: return Layout<kBF16>::kTileBytes;
    case LPAR_CODEC_FP8_E4M3: return Layout<kFP8>::kTileBytes;
    case LPAR_CODEC_INT4: return Layout<kINT4>::kTileBytes;
    case LPAR_CODEC_INT3: return Layout<kINT3>::kTileBytes;
    case LPAR_CODEC_MXFP4: return Layout<kMXFP4>::kTileBytes;
    default: return 0;
    }
}

LPAR_API size_t lpar_wire_bytes(lpar_codec_t codec, size_t n) { return (n / kTileElems) * lpar_tile_bytes(codec); }

LPAR_API size_t lpar_workspace_bytes(int N, size_t n, lpar_codec_t codec) {
    if (N < 1 || N > kMaxRanks || !codec_ok(codec)) return 0;
    if (codec == LPAR_CODEC_BF16) return lpar_wire_bytes(LPAR_CODEC_BF16, n);
    return (size_t)(N + 1) * lpar_wire_bytes(codec, n);
}

LPAR_API lpar_codec_t lpar_effective_codec(size_t n, lpar_codec_t codec, const lpar_options_t *opts) {
    const size_t thr = opts ? opts->min_quant_bytes : 0;
    if (codec != LPAR_CODEC_BF16 && 2 * n < thr) return LPAR_CODEC_BF16;
    return codec;
}

LPAR_API const char *lpar_status_string(lpar_status_t s) {
    switch (s) {
    case LPAR_OK: return "ok";
    case LPAR_ERR_INVALID_ARG: return "invalid argument";
    case LPAR_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case LPAR_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case LPAR_ERR_UNSUPPORTED: return "unsupported codec or schedule";
    case LPAR_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

LPAR_API lpar_status_t lpar_quantize(const void *in_bf16, size_t n, lpar_codec_t codec, void *wire,
                                     cudaStream_t stream) {
    NvtxRange trace("lpar_quantize");
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    if (n % kTileElems != 0 || n / kTileElems > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (n == 0) return LPAR_OK;
    if (!in_bf16 || !wire) return LPAR_ERR_INVALID_ARG;
    if (!aligned16(in_bf16) || !aligned16(wire)) return LPAR_ERR_MISALIGNED;
    const size_t tiles = n / kTileElems;
    OutPtrs w{};
    w.p[0] = static_cast<uint8_t *>(wire);
    if (codec == LPAR_CODEC_BF16) {
        launch_broadcast(static_cast<const uint8_t *>(in_bf16), w, 1, 2 * n, stream);
    } else {
        InPtrs in{};
        in.p[0] = static_cast<const uint8_t *>(in_bf16);
        launch_quantize(codec, in, w, 1, tiles, stream);
    }
    return launch_status();
}

LPAR_API lpar_status_t lpar_reduce(const void *const *wires, int N, size_t tile_begin, size_t tile_count,
                                   lpar_codec_t codec, void *wire_out, cudaStream_t stream) {
    NvtxRange trace("lpar_reduce");
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    if (N < 1 || N > kMaxRanks || !wires) return LPAR_ERR_INVALID_ARG;
    if (tile_begin + tile_count < tile_begin || tile_count > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (tile_count == 0) return LPAR_OK;
    if (!wire_out) return LPAR_ERR_INVALID_ARG;
    InPtrs w{};
    for (int r = 0; r < N; ++r) {
        if (!wires[r]) return LPAR_ERR_INVALID_ARG;
        if (!aligned16(wires[r])) return LPAR_ERR_MISALIGNED;
        w.p[r] = static_cast<const uint8_t *>(wires[r]);
    }
    if (!aligned16(wire_out)) return LPAR_ERR_MISALIGNED;
    OutPtrs none{};
    uint8_t *g = static_cast<uint8_t *>(wire_out);
    if (codec == LPAR_CODEC_BF16) {
        const size_t v_per_tile = (size_t)kTileElems * 2 / 16;
        launch_bf16_reduce<false>(w, N, g, none, tile_begin * v_per_tile, (tile_begin + tile_count) * v_per_tile,
                                  stream);
    } else {
        launch_reduce<false>(codec, w, N, g, none, tile_begin, tile_begin + tile_count, stream);
    }
    return launch_status();
}

LPAR_API lpar_status_t lpar_decode(const void *wire, size_t n, lpar_codec_t codec, void *out_bf16,
                                   cudaStream_t stream) {
    NvtxRange trace("lpar_decode");
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    if (n % kTileElems != 0 || n / kTileElems > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (n == 0) return LPAR_OK;
    if (!wire || !out_bf16) return LPAR_ERR_INVALID_ARG;
    if (!aligned16(wire) || !aligned16(out_bf16)) return LPAR_ERR_MISALIGNED;
    OutPtrs o{};
    o.p[0] = static_cast<uint8_t *>(out_bf16);
    if (codec == LPAR_CODEC_BF16) launch_broadcast(static_cast<const uint8_t *>(wire), o, 1, 2 * n, stream);
    else launch_decode(codec, static_cast<const uint8_t *>(wire), o, 1, n / kTileElems, stream);
    return launch_status();
}

LPAR_API lpar_status_t lpar_allreduce(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                      void *const *out, void *workspace, size_t workspace_bytes,
                                      const lpar_options_t *opts, cudaStream_t stream) {
    NvtxRange trace("lpar_allreduce");
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    int schedule = opts ? (int)opts->schedule : (int)LPAR_SCHEDULE_AUTO;
    if (schedule != LPAR_SCHEDULE_AUTO && schedule != LPAR_SCHEDULE_FUSED &&
        schedule != LPAR_SCHEDULE_THREE_STAGE && schedule != LPAR_SCHEDULE_SINGLE_PASS &&
        schedule != LPAR_SCHEDULE_ONE_SHOT)
        return LPAR_ERR_UNSUPPORTED;
    if (schedule == LPAR_SCHEDULE_AUTO) schedule = LPAR_SCHEDULE_SINGLE_PASS;
    if (N < 1 || N > kMaxRanks || n % kTileElems != 0 || n / kTileElems > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (n == 0) return LPAR_OK;
    if (!inputs || !out || !workspace) return LPAR_ERR_INVALID_ARG;
    InPtrs in{};
    OutPtrs o{};
    for (int r = 0; r < N; ++r) {
        if (!inputs[r] || !out[r]) return LPAR_ERR_INVALID_ARG;
        if (!aligned16(inputs[r]) || !aligned16(out[r])) return LPAR_ERR_MISALIGNED;
        in.p[r] = static_cast<const uint8_t *>(inputs[r]);
        o.p[r] = static_cast<uint8_t *>(out[r]);
    }
    if (!aligned16(workspace)) return LPAR_ERR_MISALIGNED;
    const lpar_codec_t eff = lpar_effective_codec(n, codec, opts);
    if (workspace_bytes < lpar_workspace_bytes(N, n, eff)) return LPAR_ERR_WORKSPACE_TOO_SMALL;
    const size_t tiles = n / kTileElems;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (schedule == LPAR_SCHEDULE_ONE_SHOT) {
        // every rank reduces all N stage-1 wires (the first N wires of the workspace)
        OutPtrs w1{};
        const size_t wb1 = eff == LPAR_CODEC_BF16 ? 0 : lpar_wire_bytes(eff, n);
        for (int r = 0; r < N; ++r) w1.p[r] = ws + (size_t)r * wb1;
        if (opts && opts->stage_events[0]) cudaEventRecord(opts->stage_events[0], stream);
        if (!launch_reduce_to_bf16(eff, in, w1, o, N, tiles, true, stream)) return LPAR_ERR_CUDA;
        if (opts && opts->stage_events[1]) cudaEventRecord(opts->stage_events[1], stream);
        return launch_status();
    }
    const bool fused = schedule != LPAR_SCHEDULE_THREE_STAGE;   // BF16: fused and single-pass coincide
    auto mark = [&](int i) {
        if (opts && opts->stage_events[i]) cudaEventRecord(opts->stage_events[i], stream);
    };

    if (eff == LPAR_CODEC_BF16) {
        // the wire of every rank is its input; the gathered wire is the workspace
        const size_t nvec = 2 * n / 16;
        mark(0);
        mark(1);
        if (fused) {
            launch_bf16_reduce<true>(in, N, ws, o, 0, nvec, stream);
            mark(2);
        } else {
            launch_bf16_reduce<false>(in, N, ws, o, 0, nvec, stream);
            if (cudaGetLastError() != cudaSuccess) return LPAR_ERR_CUDA;
            mark(2);
            launch_broadcast(ws, o, N, 2 * n, stream);
            mark(3);
        }
        return launch_status();
    }

    const size_t wb = lpar_wire_bytes(eff, n);
    OutPtrs wires{};
    InPtrs wires_in{};
    for (int r = 0; r < N; ++r) {
        wires.p[r] = ws + (size_t)r * wb;
        wires_in.p[r] = ws + (size_t)r * wb;
    }
    uint8_t *gather = ws + (size_t)N * wb;
    mark(0);
    if (schedule == LPAR_SCHEDULE_SINGLE_PASS) {
        if (!launch_single(eff, in, wires, N, gather, o, tiles, stream)) return LPAR_ERR_CUDA;
        mark(1);
        return launch_status();
    }
    launch_quantize(eff, in, wires, N, tiles, stream);
    if (cudaGetLastError() != cudaSuccess) return LPAR_ERR_CUDA;
    mark(1);
    if (fused) {
        launch_reduce<true>(eff, wires_in, N, gather, o, 0, tiles, stream);
        mark(2);
    } else {
        launch_reduce<false>(eff, wires_in, N, gather, o, 0, tiles, stream);
        if (cudaGetLastError() != cudaSuccess) return LPAR_ERR_CUDA;
        mark(2);
        launch_decode(eff, gather, o, N, tiles, stream);
        mark(3);
    }
    return launch_status();
}
