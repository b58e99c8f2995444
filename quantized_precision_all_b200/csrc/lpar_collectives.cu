// lpar_collectives.cu -- sm_100a kernels and C ABI of the standalone
// low-precision collectives ("RCCLX: Innovating GPU communications on AMD
// platforms", Low-Precision Collectives: the quantised wire carries the other
// collectives too, compute stays in FP32) and of the one-shot all-reduce (its
// Direct Data Access section: the flat algorithm, where every rank reduces all
// inputs itself).
//
// Every collective quantises each rank's message once into that rank's wire
// (the transmitted data, written to HBM), then:
//   reduce-scatter   sums the dequantised wires of each tile in FP32 in rank
//                    order from +0 and rounds once to BF16 into the tile's
//                    shard owner (floor partition, as the all-reduce's shards)
//   one-shot all-reduce   the same sum into every rank's output
//   all-gather       decodes rank r's wire into every rank's output at r * m
//   all-to-all       decodes segment j of rank r's wire into rank j's output at
//                    r * m
// The BF16 passthrough (below the threshold, or codec BF16) moves the BF16
// values themselves.  Each quantising collective is one persistent kernel of
// the single-pass shape (see lpar_kernels.cu): a CTA quantises a 4-tile chunk,
// then reduces or decodes it while cp.async prefetches the next chunk.  The
// reductions come in a warp-local and a CTA-wide form (picked by codec, N and
// size), the all-gather and all-to-all send their outputs by bulk copies.
#include "lpar.h"
#include "lpar_codec.cuh"
#include "lpar_tiles.cuh"

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

namespace lpar {

// Floor partition of T tiles into N shards: shard j is [jT/N, (j+1)T/N), and
// tile t belongs to shard ((t + 1) N - 1) / T (the largest j with jT/N <= t).
__host__ __device__ __forceinline__ size_t shard_begin(int j, size_t T, int N) {
    return (size_t)j * T / (size_t)N;
}
__host__ __device__ __forceinline__ int shard_of(size_t t, size_t T, int N) {
    return (int)(((t + 1) * (size_t)N - 1) / T);
}

// Stage 1 of one rank's chunk from the staged BF16 (thread t's block) into the
// wire; with WANT_V the decoded block also goes to `sink`.
template <int C, bool WANT_V, class Sink>
__device__ __forceinline__ void quantize_staged_block(const uint8_t *stage, uint8_t *wire_tile, int t,
                                                      const Sink &sink) {
    uint32_t x16[16];
    stage_read(stage, t, x16);
    float x[32];
#pragma unroll
    for (int k = 0; k < 16; ++k) { x[2 * k] = bf16lo(x16[k]); x[2 * k + 1] = bf16hi(x16[k]); }
    const float a = absmax_bf16x32(x16);
    Packed<C> p;
    encode<C, false, WANT_V>(x, a, p, sink);
    store_block(wire_tile, t % kBlocksPerTile, p);
}

// ---------------------------------------------------------------------------
// Reduce-scatter (ALL = false) and one-shot all-reduce (ALL = true), quantising
// codecs.  Per chunk: stage 1 of every rank (prefetching the next rank's BF16
// chunk), then each thread reads back the N wire blocks it wrote, sums them
// and rounds to BF16; the staged chunk goes to the shard owners or to all.
// ---------------------------------------------------------------------------
template <int C, int N, bool ALL>
__global__ void __launch_bounds__(kThreads, 4) k_reduce_bf16_single(const __grid_constant__ InPtrs in,
                                                                    const __grid_constant__ OutPtrs wire,
                                                                    const __grid_constant__ OutPtrs out,
                                                                    size_t tiles, unsigned chunks) {
    __shared__ __align__(128) uint8_t stage_in[2][kStageBytes];
    __shared__ uint8_t *s_dst[kTilesPerCta];
    const int t = threadIdx.x;
    unsigned c = blockIdx.x;
    if (c < chunks) {
        const size_t tile0 = (size_t)c * kTilesPerCta;
        stage_load_chunk(stage_in[0], in.p[0] + tile0 * (kTileElems * 2),
                         (int)min((size_t)kTilesPerCta, tiles - tile0));
    }
    cp_async_commit();
    int buf = 0;
    for (; c < chunks; c += gridDim.x) {
        const size_t tile0 = (size_t)c * kTilesPerCta;
        const int ntiles = (int)min((size_t)kTilesPerCta, tiles - tile0);
        const bool active = t < ntiles * kBlocksPerTile;
        const size_t tile = tile0 + t / kBlocksPerTile;
        const int b = t % kBlocksPerTile;
#pragma unroll 1
        for (int r = 0; r < N; ++r) {
            const unsigned cn = (r + 1 < N) ? c : c + gridDim.x;
            if (cn < chunks) {
                const size_t tn = (size_t)cn * kTilesPerCta;
                stage_load_chunk(stage_in[buf ^ 1], in.p[(r + 1 < N) ? r + 1 : 0] + tn * (kTileElems * 2),
                                 (int)min((size_t)kTilesPerCta, tiles - tn));
            }
            cp_async_commit();
            cp_async_wait_prev();
            __syncthreads();
            if (active)
                quantize_staged_block<C, false>(stage_in[buf], wire.p[r] + tile * Layout<C>::kTileBytes, t, NoSink{});
            __syncthreads();                               // stage_in[buf] is refilled next
            buf ^= 1;
        }
        // The buffer of the last rank's chunk is free until the next chunk's
        // first prefetch (after the closing barrier): it stages the output.
        uint8_t *stage_out = stage_in[buf ^ 1];
        if (active) {
            float acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0.0f;    // +0.0f, then ranks in ascending order
#pragma unroll
            for (int r = 0; r < N; ++r) {
                Packed<C> p;
                load_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
                accumulate<C>(p, acc);
            }
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = pack_bf16x2(acc[2 * k], acc[2 * k + 1]);
            stage_write(stage_out, t, o);
        }
        if (!ALL && t < ntiles) {
            const size_t tt = tile0 + t;
            const int j = shard_of(tt, tiles, N);
            s_dst[t] = out.p[j] + (tt - shard_begin(j, tiles, N)) * (kTileElems * 2);
        }
        __syncthreads();
        if (ALL) stage_to_outputs(stage_out, out, N, tile0 * (kTileElems * 2), ntiles);
        else stage_to_tile_dsts(stage_out, s_dst, ntiles);
        __syncthreads();                                   // stage_out and s_dst are reused next chunk
    }
}

// The warp-local form of the reductions (see k_allreduce_single_warp): every
// warp copies, encodes, reduces and stores only its own half tile of the
// chunk, so no CTA barrier is needed; a ring of three stages per warp, the
// BF16 sums staged in place of the last rank's input.
template <int C, int N, bool ALL>
__global__ void __launch_bounds__(kThreads, 4) k_reduce_bf16_warp(const __grid_constant__ InPtrs in,
                                                                  const __grid_constant__ OutPtrs wire,
                                                                  const __grid_constant__ OutPtrs out,
                                                                  size_t tiles, unsigned chunks) {
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
            const int nb = buf + 1 == S ? 0 : buf + 1;
            const unsigned cn = (r + 1 < N) ? c : c + gridDim.x;
            if (cn < chunks && has(cn))
                warp_load(ring + nb * kStageBytes,
                          in.p[(r + 1 < N) ? r + 1 : 0] + (size_t)cn * kTilesPerCta * (kTileElems * 2), w, lane);
            cp_async_commit();
            cp_async_wait_prev();
            __syncwarp();                                  // the warp's item landed
            if (active)
                quantize_staged_block<C, false>(ring + buf * kStageBytes, wire.p[r] + tile * Layout<C>::kTileBytes,
                                                t, NoSink{});
            last = buf;
            buf = nb;
        }
        uint8_t *const so = ring + last * kStageBytes;
        if (active) {
            float acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0.0f;    // +0.0f, then ranks in ascending order
#pragma unroll
            for (int r = 0; r < N; ++r) {
                Packed<C> p;
                load_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
                accumulate<C>(p, acc);
            }
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = pack_bf16x2(acc[2 * k], acc[2 * k + 1]);
            stage_write(so, t, o);
        }
        __syncwarp();
        if (active) {
            if (ALL) {
                warp_to_outputs(so, out, N, tile0 * (kTileElems * 2), w, lane);
            } else {
                const int j = shard_of(tile, tiles, N);
                warp_to_dst(so, out.p[j] + (tile - shard_begin(j, tiles, N)) * (kTileElems * 2) + (w & 1) * kWarpBytes,
                            w, lane);
            }
        }
    }
}

// The rank-parallel tile form of the reductions (small messages; see
// k_allreduce_tile): one tile per CTA, the N ranks' tiles copied into shared
// memory and their N x 64 block encodes spread over the threads; after one
// barrier threads 0..63 read back the N wire blocks of their block, sum them in
// rank order from +0.0f and round once to BF16 into rank 0's region, which all
// threads store to the shard owner (ALL = false) or to every rank.
template <int C, int N, bool ALL>
__global__ void __launch_bounds__(kThreads) k_reduce_bf16_tile(const __grid_constant__ InPtrs in,
                                                               const __grid_constant__ OutPtrs wire,
                                                               const __grid_constant__ OutPtrs out, size_t tiles) {
    constexpr int kTileBytesBf16 = kTileElems * 2;
    __shared__ __align__(128) uint8_t stage[N * kTileBytesBf16];
    const int t = threadIdx.x;
    const size_t tile = blockIdx.x;
#pragma unroll
    for (int r = 0; r < N; ++r)
        cp_async16(stage + r * kTileBytesBf16 + swz(t >> 2, t & 3), in.p[r] + tile * kTileBytesBf16 + 16 * t);
    cp_async_commit();
    cp_async_wait_all_groups();
    __syncthreads();
#pragma unroll
    for (int k = 0; k < (N + 3) / 4; ++k) {
        const int idx = t + kThreads * k, r = idx >> 6, b = idx & 63;
        if (r < N)
            quantize_staged_block<C, false>(stage + r * kTileBytesBf16, wire.p[r] + tile * Layout<C>::kTileBytes, b,
                                            NoSink{});
    }
    __syncthreads();                                             // wire blocks visible; rank 0's region free
    if (t < kBlocksPerTile) {
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.0f;              // +0.0f, then ranks in ascending order
#pragma unroll
        for (int r = 0; r < N; ++r) {
            Packed<C> p;
            load_block(wire.p[r] + tile * Layout<C>::kTileBytes, t, p);
            accumulate<C>(p, acc);
        }
        uint32_t o[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = pack_bf16x2(acc[2 * k], acc[2 * k + 1]);
        stage_write(stage, t, o);
    }
    __syncthreads();
    const uint4 d = *reinterpret_cast<const uint4 *>(stage + swz(t >> 2, t & 3));
    if (ALL) {
#pragma unroll
        for (int r = 0; r < N; ++r) *reinterpret_cast<uint4 *>(out.p[r] + tile * kTileBytesBf16 + 16 * t) = d;
    } else {
        const int j = shard_of(tile, tiles, N);
        *reinterpret_cast<uint4 *>(out.p[j] + (tile - shard_begin(j, tiles, N)) * kTileBytesBf16 + 16 * t) = d;
    }
}

// BF16 passthrough of the reductions: one tile (256 x 16 B) per CTA step, the
// FP32 sum in rank order rounded once.  The shard owner advances with the
// tile index (tiles are visited in increasing order), so no division per tile.
template <int N, bool ALL>
__global__ void __launch_bounds__(kThreads) k_bf16_reduce_to(const __grid_constant__ InPtrs in,
                                                             const __grid_constant__ OutPtrs out, size_t tiles) {
    const int t = threadIdx.x;
    size_t tile = blockIdx.x;
    if (tile >= tiles) return;
    int j = ALL ? 0 : shard_of(tile, tiles, N);
    size_t jb = ALL ? 0 : shard_begin(j, tiles, N), je = ALL ? 0 : shard_begin(j + 1, tiles, N);
    for (; tile < tiles; tile += gridDim.x) {
        if (!ALL) {
            while (tile >= je) { ++j; jb = je; je = shard_begin(j + 1, tiles, N); }
        }
        const size_t off = tile * (kTileElems * 2) + 16 * (size_t)t;
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
#pragma unroll
        for (int r = 0; r < N; ++r) {
            const uint4 x = *reinterpret_cast<const uint4 *>(in.p[r] + off);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc[2 * k] = __fadd_rn(acc[2 * k], bf16lo(w[k]));
                acc[2 * k + 1] = __fadd_rn(acc[2 * k + 1], bf16hi(w[k]));
            }
        }
        const uint4 o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        if (ALL) {
#pragma unroll
            for (int r = 0; r < N; ++r) *reinterpret_cast<uint4 *>(out.p[r] + off) = o;
        } else {
            *reinterpret_cast<uint4 *>(out.p[j] + (tile - jb) * (kTileElems * 2) + 16 * (size_t)t) = o;
        }
    }
}

// ---------------------------------------------------------------------------
// All-gather (A2A = false) and all-to-all (A2A = true), quantising codecs.
// Work items (chunk c, rank r) of the ranks' messages (`tiles` tiles each);
// the next item's BF16 chunk is prefetched while the current one is encoded.
// The block's decoded values come from the encoder's registers (the value the
// receiver decodes from the wire, which is written as the transmitted data).
// seg_tiles is the segment length m / 2048 (all-gather: the whole message).
// ---------------------------------------------------------------------------
// Stages in the gather ring (measured on B200, one process timing the
// variants alternately): the all-gather's time does not move from three to six
// stages, so it keeps three (four CTAs per SM); the all-to-all, whose copies
// are one tile each, gains from deeper rings -- five stages for FP8 (9% at
// N = 8), four for the others (2-4%).
template <int C, bool A2A>
__host__ __device__ constexpr int gather_stages() { return A2A ? (C == kFP8 ? 5 : 4) : 3; }
template <int C, bool A2A>
__host__ __device__ constexpr int gather_smem() { return gather_stages<C, A2A>() * kStageBytes; }
template <int C, bool A2A>
__host__ __device__ constexpr int gather_min_ctas() {       // CTAs per SM the ring's shared memory allows
    return gather_stages<C, A2A>() == 3 ? 4 : (gather_stages<C, A2A>() == 4 ? 3 : 2);
}

template <int C, bool A2A>
__global__ void __launch_bounds__(kThreads, gather_min_ctas<C, A2A>())
    k_gather_single(const __grid_constant__ InPtrs in, const __grid_constant__ OutPtrs wire,
                    const __grid_constant__ OutPtrs out, size_t tiles, size_t seg_tiles, unsigned chunks, int N) {
    // A ring of S BF16 stages.  Item i is staged in stage i % S while item
    // i + 1 is prefetched into the next stage; its decoded chunk replaces its
    // input in place (in element order; each thread writes only the 64-B
    // region it read) and leaves through bulk copies issued by lanes of warp 0,
    // which read the stage while the following items are encoded.  Stage i % S
    // is refilled by item i + S - 1's prefetch, so before the barrier that
    // closes item i + S - 2 those lanes wait until at most the S - 3 newest
    // groups of copies are still reading.
    constexpr int S = gather_stages<C, A2A>();
    static_assert(S >= 3 && S <= 5, "ring of three to five stages");
    extern __shared__ __align__(1024) uint8_t ring[];
    const int t = threadIdx.x;
    unsigned c = blockIdx.x;
    if (c >= chunks) return;
    int r = 0;
    stage_load_chunk(ring, in.p[0] + (size_t)c * kTilesPerCta * (kTileElems * 2),
                     (int)min((size_t)kTilesPerCta, tiles - (size_t)c * kTilesPerCta));
    cp_async_commit();
    int buf = 0;
    while (c < chunks) {
        unsigned cn = c;
        int rn = r + 1;
        if (rn == N) { rn = 0; cn += gridDim.x; }
        const int nb = buf + 1 == S ? 0 : buf + 1;
        if (cn < chunks) {
            const size_t tn = (size_t)cn * kTilesPerCta;
            stage_load_chunk(ring + nb * kStageBytes, in.p[rn] + tn * (kTileElems * 2),
                             (int)min((size_t)kTilesPerCta, tiles - tn));
        }
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();                                   // item landed
        uint8_t *const st = ring + buf * kStageBytes;
        const size_t tile0 = (size_t)c * kTilesPerCta;
        const int ntiles = (int)min((size_t)kTilesPerCta, tiles - tile0);
        if (t < ntiles * kBlocksPerTile)
            quantize_staged_block<C, true>(st, wire.p[r] + (tile0 + t / kBlocksPerTile) * Layout<C>::kTileBytes, t,
                                           StageSinkLinear{st, t});
        fence_async_smem();
        if (t < 32) bulk_wait_read<S - 3>();
        __syncthreads();                                   // decoded chunk complete
        if (A2A) {
            if (t < ntiles) {                              // tile t of rank r's message -> its segment's rank
                const size_t tt = tile0 + t;
                const size_t j = tt / seg_tiles;
                bulk_store(out.p[j] + ((size_t)r * seg_tiles + (tt - j * seg_tiles)) * (kTileElems * 2),
                           st + t * (kTileElems * 2), kTileElems * 2);
            }
        } else if (t < N) {                                // the chunk to output t at rank r's place
            bulk_store(out.p[t] + ((size_t)r * tiles + tile0) * (kTileElems * 2), st,
                       (unsigned)ntiles * (kTileElems * 2));
        }
        if (t < 32) bulk_commit();
        buf = nb;
        c = cn;
        r = rn;
    }
    if (t < 32) bulk_wait_read<0>();                  // the stage outlives no copy that reads it
}

// BF16 passthrough of all-gather / all-to-all: copies, one tile of one rank per
// CTA step (grid.y = rank).  The all-to-all segment advances with the tile.
template <bool A2A>
__global__ void __launch_bounds__(kThreads) k_bf16_gather(const __grid_constant__ InPtrs in,
                                                          const __grid_constant__ OutPtrs out, size_t tiles,
                                                          size_t seg_tiles, int N) {
    const int t = threadIdx.x;
    const int r = blockIdx.y;
    size_t tile = blockIdx.x;
    if (tile >= tiles) return;
    size_t j = A2A ? tile / seg_tiles : 0, je = (j + 1) * seg_tiles;
    for (; tile < tiles; tile += gridDim.x) {
        const uint4 d = *reinterpret_cast<const uint4 *>(in.p[r] + tile * (kTileElems * 2) + 16 * (size_t)t);
        if (A2A) {
            while (tile >= je) { ++j; je += seg_tiles; }
            const size_t dt = (size_t)r * seg_tiles + (tile - (je - seg_tiles));
            *reinterpret_cast<uint4 *>(out.p[j] + dt * (kTileElems * 2) + 16 * (size_t)t) = d;
        } else {
            const size_t off = ((size_t)r * tiles + tile) * (kTileElems * 2) + 16 * (size_t)t;
#pragma unroll
            for (int k = 0; k < kMaxRanks; ++k)
                if (k < N) *reinterpret_cast<uint4 *>(out.p[k] + off) = d;
        }
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers (arguments validated by the callers).
// ---------------------------------------------------------------------------
static inline unsigned persistent_grid(unsigned chunks, unsigned resident) {
    return std::min<unsigned>(chunks, std::max<unsigned>(1u, resident ? resident : 148u * 4u));
}

// Which form of the reductions runs (measured on B200, the forms timed
// alternately in one process): the rank-parallel tile form up to
// kTileFormMaxTiles tiles per rank; above, the warp-local form below 128 MiB of input for
// every codec but FP8 (5-10% faster) and, for the reduce-scatter, for INT3 at
// every size (6-9%) and for INT4 and MXFP4 from four ranks on (8% at N = 8);
// the CTA-wide form for FP8, for the one-shot from 128 MiB (4-9%) and for the
// reduce-scatter of INT4 and MXFP4 with fewer ranks (3-9%).
static inline bool rs_warp_form(int C, int N, bool ALL, size_t in_bytes) {
    if (C == kFP8) return false;
    if (in_bytes < ((size_t)128 << 20)) return true;
    if (ALL) return false;
    return C == kINT3 || N >= 4;
}

template <int C, int N, bool ALL>
static bool launch_rb_cna(const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, size_t tiles, cudaStream_t st) {
    if (tiles <= kTileFormMaxTiles<C>()) {
        k_reduce_bf16_tile<C, N, ALL><<<(unsigned)tiles, kThreads, 0, st>>>(in, wire, out, tiles);
        return true;
    }
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    if (rs_warp_form(C, N, ALL, (size_t)N * tiles * (kTileElems * 2))) {
        constexpr int smem = 3 * kStageBytes;
        if (!allow_dynamic_smem<k_reduce_bf16_warp<C, N, ALL>>(smem)) return false;
        const unsigned grid = persistent_grid(chunks, resident_ctas<k_reduce_bf16_warp<C, N, ALL>>(smem));
        k_reduce_bf16_warp<C, N, ALL><<<grid, kThreads, smem, st>>>(in, wire, out, tiles, chunks);
        return true;
    }
    const unsigned grid = persistent_grid(chunks, resident_ctas<k_reduce_bf16_single<C, N, ALL>>());
    k_reduce_bf16_single<C, N, ALL><<<grid, kThreads, 0, st>>>(in, wire, out, tiles, chunks);
    return true;
}

template <int N, bool ALL>
static bool launch_rb_na(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, size_t tiles,
                         cudaStream_t st) {
    switch (codec) {
    case kINT4: return launch_rb_cna<kINT4, N, ALL>(in, wire, out, tiles, st);
    case kINT3: return launch_rb_cna<kINT3, N, ALL>(in, wire, out, tiles, st);
    case kFP8: return launch_rb_cna<kFP8, N, ALL>(in, wire, out, tiles, st);
    case kMXFP4: return launch_rb_cna<kMXFP4, N, ALL>(in, wire, out, tiles, st);
    default: {
        const unsigned grid = (unsigned)std::min<size_t>(tiles, (size_t)1 << 20);
        k_bf16_reduce_to<N, ALL><<<grid, kThreads, 0, st>>>(in, out, tiles);
        return true;
    }
    }
}

template <bool ALL>
static bool launch_rb_a(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N, size_t tiles,
                        cudaStream_t st) {
    switch (N) {
    case 1: return launch_rb_na<1, ALL>(codec, in, wire, out, tiles, st);
    case 2: return launch_rb_na<2, ALL>(codec, in, wire, out, tiles, st);
    case 3: return launch_rb_na<3, ALL>(codec, in, wire, out, tiles, st);
    case 4: return launch_rb_na<4, ALL>(codec, in, wire, out, tiles, st);
    case 5: return launch_rb_na<5, ALL>(codec, in, wire, out, tiles, st);
    case 6: return launch_rb_na<6, ALL>(codec, in, wire, out, tiles, st);
    case 7: return launch_rb_na<7, ALL>(codec, in, wire, out, tiles, st);
    case 8: return launch_rb_na<8, ALL>(codec, in, wire, out, tiles, st);
    default: return false;
    }
}

bool launch_reduce_to_bf16(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N,
                           size_t tiles, bool all, cudaStream_t st) {
    return all ? launch_rb_a<true>(codec, in, wire, out, N, tiles, st)
               : launch_rb_a<false>(codec, in, wire, out, N, tiles, st);
}

template <int C, bool A2A>
static bool launch_gather_c(const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N, size_t tiles,
                            size_t seg_tiles, cudaStream_t st) {
    constexpr int smem = gather_smem<C, A2A>();
    if (!allow_dynamic_smem<k_gather_single<C, A2A>>(smem)) return false;
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    unsigned grid = persistent_grid(chunks, resident_ctas<k_gather_single<C, A2A>>(smem));
    // The all-gather writes N outputs per item: from 64 MiB of input, fewer
    // CTAs (fewer concurrent output streams) write faster -- two per SM up to
    // three ranks, one from four (measured on B200, 4-8% at 64-256 MiB); with
    // eight ranks the counts measured alike (within 2%) and all CTAs stay.
    if (!A2A && N < 8 && (size_t)N * tiles * (kTileElems * 2) >= ((size_t)64 << 20)) {
        const unsigned sms = sm_count();
        if (sms) grid = std::min<unsigned>(grid, sms * (N <= 3 ? 2u : 1u));
    }
    k_gather_single<C, A2A><<<grid, kThreads, smem, st>>>(in, wire, out, tiles, seg_tiles, chunks, N);
    return true;
}

template <bool A2A>
static bool launch_gather(int codec, const InPtrs &in, const OutPtrs &wire, const OutPtrs &out, int N,
                          size_t tiles, size_t seg_tiles, cudaStream_t st) {
    switch (codec) {
    case kINT4: return launch_gather_c<kINT4, A2A>(in, wire, out, N, tiles, seg_tiles, st);
    case kINT3: return launch_gather_c<kINT3, A2A>(in, wire, out, N, tiles, seg_tiles, st);
    case kFP8: return launch_gather_c<kFP8, A2A>(in, wire, out, N, tiles, seg_tiles, st);
    case kMXFP4: return launch_gather_c<kMXFP4, A2A>(in, wire, out, N, tiles, seg_tiles, st);
    default: {
        const dim3 grid((unsigned)std::min<size_t>(tiles, (size_t)1 << 20), (unsigned)N);
        k_bf16_gather<A2A><<<grid, kThreads, 0, st>>>(in, out, tiles, seg_tiles, N);
        return true;
    }
    }
}

}  // namespace lpar

using namespace lpar;

// ---------------------------------------------------------------------------
// The C ABI of the collectives.
// ---------------------------------------------------------------------------
LPAR_API size_t lpar_collective_workspace_bytes(lpar_collective_t op, int N, size_t n, lpar_codec_t codec) {
    if (N < 1 || N > kMaxRanks || !codec_ok(codec)) return 0;
    switch (op) {
    case LPAR_OP_ALLREDUCE: return lpar_workspace_bytes(N, n, codec);
    case LPAR_OP_ALLREDUCE_F32:
        return codec == LPAR_CODEC_BF16 ? 4 * n : (size_t)(N + 1) * lpar_wire_bytes(codec, n);
    case LPAR_OP_REDUCE_SCATTER:
    case LPAR_OP_ALL_GATHER: return codec == LPAR_CODEC_BF16 ? 0 : (size_t)N * lpar_wire_bytes(codec, n);
    case LPAR_OP_ALL_TO_ALL: return codec == LPAR_CODEC_BF16 ? 0 : (size_t)N * lpar_wire_bytes(codec, (size_t)N * n);
    default: return 0;
    }
}

// Shared validation of the three collectives.  `n_msg` is the per-rank message
// in elements (reduce-scatter: n; all-gather: m; all-to-all: N * m).
static lpar_status_t collective_setup(lpar_collective_t op, const void *const *inputs, int N, size_t size,
                                      lpar_codec_t codec, void *const *out, void *workspace,
                                      size_t workspace_bytes, const lpar_options_t *opts, InPtrs &in, OutPtrs &o,
                                      OutPtrs &wires, lpar_codec_t &eff, size_t &n_msg) {
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    if (N < 1 || N > kMaxRanks || size % kTileElems != 0) return LPAR_ERR_INVALID_ARG;
    if (size / kTileElems > kMaxTiles) return LPAR_ERR_INVALID_ARG;   // also keeps N * size from wrapping
    n_msg = op == LPAR_OP_ALL_TO_ALL ? (size_t)N * size : size;
    if (n_msg / kTileElems > kMaxTiles) return LPAR_ERR_INVALID_ARG;
    if (n_msg == 0) return LPAR_OK;
    if (!inputs || !out) return LPAR_ERR_INVALID_ARG;
    for (int r = 0; r < N; ++r) {
        if (!inputs[r] || !out[r]) return LPAR_ERR_INVALID_ARG;
        if (!aligned16(inputs[r]) || !aligned16(out[r])) return LPAR_ERR_MISALIGNED;
        in.p[r] = static_cast<const uint8_t *>(inputs[r]);
        o.p[r] = static_cast<uint8_t *>(out[r]);
    }
    eff = lpar_effective_codec(n_msg, codec, opts);
    const size_t need = lpar_collective_workspace_bytes(op, N, size, eff);
    if (need) {
        if (!workspace) return LPAR_ERR_INVALID_ARG;
        if (!aligned16(workspace)) return LPAR_ERR_MISALIGNED;
        if (workspace_bytes < need) return LPAR_ERR_WORKSPACE_TOO_SMALL;
        const size_t wb = lpar_wire_bytes(eff, n_msg);
        for (int r = 0; r < N; ++r) wires.p[r] = static_cast<uint8_t *>(workspace) + (size_t)r * wb;
    }
    return LPAR_OK;
}

static inline void mark(const lpar_options_t *opts, int i, cudaStream_t stream) {
    if (opts && opts->stage_events[i]) cudaEventRecord(opts->stage_events[i], stream);
}

LPAR_API lpar_status_t lpar_reduce_scatter(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                           void *const *out, void *workspace, size_t workspace_bytes,
                                           const lpar_options_t *opts, cudaStream_t stream) {
    NvtxRange trace("lpar_reduce_scatter");
    InPtrs in{};
    OutPtrs o{}, wires{};
    lpar_codec_t eff = codec;
    size_t n_msg = 0;
    const lpar_status_t st = collective_setup(LPAR_OP_REDUCE_SCATTER, inputs, N, n, codec, out, workspace,
                                              workspace_bytes, opts, in, o, wires, eff, n_msg);
    if (st != LPAR_OK || n_msg == 0) return st;
    mark(opts, 0, stream);
    if (!launch_reduce_to_bf16(eff, in, wires, o, N, n / kTileElems, false, stream)) return LPAR_ERR_CUDA;
    mark(opts, 1, stream);
    return launch_status();
}

LPAR_API lpar_status_t lpar_all_gather(const void *const *inputs, int N, size_t m, lpar_codec_t codec,
                                       void *const *out, void *workspace, size_t workspace_bytes,
                                       const lpar_options_t *opts, cudaStream_t stream) {
    NvtxRange trace("lpar_all_gather");
    InPtrs in{};
    OutPtrs o{}, wires{};
    lpar_codec_t eff = codec;
    size_t n_msg = 0;
    const lpar_status_t st = collective_setup(LPAR_OP_ALL_GATHER, inputs, N, m, codec, out, workspace,
                                              workspace_bytes, opts, in, o, wires, eff, n_msg);
    if (st != LPAR_OK || n_msg == 0) return st;
    const size_t tiles = m / kTileElems;
    mark(opts, 0, stream);
    if (!launch_gather<false>(eff, in, wires, o, N, tiles, tiles, stream)) return LPAR_ERR_CUDA;
    mark(opts, 1, stream);
    return launch_status();
}

LPAR_API lpar_status_t lpar_all_to_all(const void *const *inputs, int N, size_t m, lpar_codec_t codec,
                                       void *const *out, void *workspace, size_t workspace_bytes,
                                       const lpar_options_t *opts, cudaStream_t stream) {
    NvtxRange trace("lpar_all_to_all");
    InPtrs in{};
    OutPtrs o{}, wires{};
    lpar_codec_t eff = codec;
    size_t n_msg = 0;
    const lpar_status_t st = collective_setup(LPAR_OP_ALL_TO_ALL, inputs, N, m, codec, out, workspace,
                                              workspace_bytes, opts, in, o, wires, eff, n_msg);
    if (st != LPAR_OK || n_msg == 0) return st;
    mark(opts, 0, stream);
    if (!launch_gather<true>(eff, in, wires, o, N, n_msg / kTileElems, m / kTileElems, stream)) return LPAR_ERR_CUDA;
    mark(opts, 1, stream);
    return launch_status();
}
