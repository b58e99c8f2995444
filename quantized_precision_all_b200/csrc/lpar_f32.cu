// lpar_f32.cu -- the all-reduce of binary32 messages on sm_100a ("RCCLX:
// Innovating GPU communications on AMD platforms", Low-Precision Collectives:
// FP32 or BF16 inputs, FP8 on the wire for up to 4:1 against FP32, compute in
// FP32) and its C ABI entry point.
//
// The tiles, codecs and stages are those of the BF16 all-reduce; the message
// blocks are binary32 (so stage 1 verifies its fast rounding like stage 2,
// since 24-bit values can sit close to a tie), and the result is the
// dequantised gathered value itself, written as binary32.  One persistent
// kernel per call (the single-pass shape of lpar_kernels.cu) with 32 KiB
// stages: two of them in 64 KiB of dynamic shared memory, and the decoded
// chunk staged in place of the last rank's input.  The uncompressed
// passthrough sums the binary32 inputs in rank order.
#include "lpar.h"
#include "lpar_codec.cuh"
#include "lpar_tiles.cuh"

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

namespace lpar {

constexpr int kSmemF32 = 2 * kStageBytesF32;            // 64 KiB

template <int C, int N>
__global__ void __launch_bounds__(kThreads, 3) k_allreduce_single_f32(const __grid_constant__ InPtrs in,
                                                                      const __grid_constant__ OutPtrs wire,
                                                                      uint8_t *gather,
                                                                      const __grid_constant__ OutPtrs out,
                                                                      size_t tiles, unsigned chunks) {
    extern __shared__ __align__(128) uint8_t smem_f32[];
    uint8_t *const stage[2] = {smem_f32, smem_f32 + kStageBytesF32};
    const int t = threadIdx.x;
    unsigned c = blockIdx.x;
    if (c >= chunks) return;
    stage_load_chunk_f32(stage[0], in.p[0] + (size_t)c * kTilesPerCta * (kTileElems * 4),
                         (int)min((size_t)kTilesPerCta, tiles - (size_t)c * kTilesPerCta));
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
                stage_load_chunk_f32(stage[buf ^ 1], in.p[(r + 1 < N) ? r + 1 : 0] + tn * (kTileElems * 4),
                                     (int)min((size_t)kTilesPerCta, tiles - tn));
            }
            cp_async_commit();
            cp_async_wait_prev();
            __syncthreads();
            if (active) {
                float x[32];
                stage_read_f32(stage[buf], t, x);
                const float a = absmax_f32x32(x);
                Packed<C> p;
                encode<C, true, false>(x, a, p, NoSink{});   // 24-bit values: verified rounding
                store_block(wire.p[r] + tile * Layout<C>::kTileBytes, b, p);
            }
            __syncthreads();                               // stage[buf] is refilled next
            buf ^= 1;
        }
        // stage[buf ^ 1] held the last rank's chunk; it is refilled only after
        // the closing barrier, so it stages the decoded chunk
        uint8_t *const so = stage[buf ^ 1];
        if (active) reduce_block<C, N, true>(wire.p, tile, b, gather, StageSinkF32{so, t});
        __syncthreads();
        stage_to_outputs_f32(so, out, N, tile0 * (kTileElems * 4), ntiles);
        __syncthreads();
    }
}

// Uncompressed passthrough: 4 binary32 values (16 B) per thread, the sum in
// rank order from +0.0f into the gathered buffer and every output.
template <int N>
__global__ void __launch_bounds__(kThreads) k_f32_reduce(const __grid_constant__ InPtrs in, float *gather,
                                                         const __grid_constant__ OutPtrs out, size_t nvec) {
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < nvec; i += (size_t)gridDim.x * kThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < N; ++r) {
            const float4 x = *reinterpret_cast<const float4 *>(in.p[r] + 16 * i);
            acc.x = __fadd_rn(acc.x, x.x);
            acc.y = __fadd_rn(acc.y, x.y);
            acc.z = __fadd_rn(acc.z, x.z);
            acc.w = __fadd_rn(acc.w, x.w);
        }
        reinterpret_cast<float4 *>(gather)[i] = acc;
#pragma unroll
        for (int r = 0; r < N; ++r) *reinterpret_cast<float4 *>(out.p[r] + 16 * i) = acc;
    }
}

// ---------------------------------------------------------------------------
// Launchers.  The 64 KiB of dynamic shared memory needs the per-kernel opt-in.
// ---------------------------------------------------------------------------
template <int C, int N>
static bool launch_f32_cn(const InPtrs &in, const OutPtrs &wire, uint8_t *g, const OutPtrs &o, size_t tiles,
                          cudaStream_t st) {
    if (!allow_dynamic_smem<k_allreduce_single_f32<C, N>>(kSmemF32)) return false;
    const unsigned chunks = (unsigned)((tiles + kTilesPerCta - 1) / kTilesPerCta);
    const unsigned res = resident_ctas<k_allreduce_single_f32<C, N>>(kSmemF32);
    const unsigned grid = std::min<unsigned>(chunks, std::max<unsigned>(1u, res ? res : 148u * 3u));
    k_allreduce_single_f32<C, N><<<grid, kThreads, kSmemF32, st>>>(in, wire, g, o, tiles, chunks);
    return true;
}

template <int C>
static bool launch_f32_c(const InPtrs &in, const OutPtrs &wire, int N, uint8_t *g, const OutPtrs &o, size_t tiles,
                         cudaStream_t st) {
    switch (N) {
    case 1: return launch_f32_cn<C, 1>(in, wire, g, o, tiles, st);
    case 2: return launch_f32_cn<C, 2>(in, wire, g, o, tiles, st);
    case 3: return launch_f32_cn<C, 3>(in, wire, g, o, tiles, st);
    case 4: return launch_f32_cn<C, 4>(in, wire, g, o, tiles, st);
    case 5: return launch_f32_cn<C, 5>(in, wire, g, o, tiles, st);
    case 6: return launch_f32_cn<C, 6>(in, wire, g, o, tiles, st);
    case 7: return launch_f32_cn<C, 7>(in, wire, g, o, tiles, st);
    case 8: return launch_f32_cn<C, 8>(in, wire, g, o, tiles, st);
    default: return false;
    }
}

template <int N>
static void launch_f32_reduce_n(const InPtrs &in, float *g, const OutPtrs &o, size_t nvec, cudaStream_t st) {
    const unsigned grid = (unsigned)std::min<size_t>((nvec + kThreads - 1) / kThreads, (size_t)148 * 32);
    k_f32_reduce<N><<<grid, kThreads, 0, st>>>(in, g, o, nvec);
}

static void launch_f32_reduce(const InPtrs &in, int N, float *g, const OutPtrs &o, size_t nvec, cudaStream_t st) {
    switch (N) {
    case 1: launch_f32_reduce_n<1>(in, g, o, nvec, st); break;
    case 2: launch_f32_reduce_n<2>(in, g, o, nvec, st); break;
    case 3: launch_f32_reduce_n<3>(in, g, o, nvec, st); break;
    case 4: launch_f32_reduce_n<4>(in, g, o, nvec, st); break;
    case 5: launch_f32_reduce_n<5>(in, g, o, nvec, st); break;
    case 6: launch_f32_reduce_n<6>(in, g, o, nvec, st); break;
    case 7: launch_f32_reduce_n<7>(in, g, o, nvec, st); break;
    case 8: launch_f32_reduce_n<8>(in, g, o, nvec, st); break;
    default: break;
    }
}

}  // namespace lpar

using namespace lpar;

LPAR_API lpar_status_t lpar_allreduce_f32(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                          void *const *out, void *workspace, size_t workspace_bytes,
                                          const lpar_options_t *opts, cudaStream_t stream) {
    NvtxRange trace("lpar_allreduce_f32");
    if (!codec_ok(codec)) return LPAR_ERR_UNSUPPORTED;
    const int schedule = opts ? (int)opts->schedule : (int)LPAR_SCHEDULE_AUTO;
    if (schedule != LPAR_SCHEDULE_AUTO && schedule != LPAR_SCHEDULE_SINGLE_PASS) return LPAR_ERR_UNSUPPORTED;
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
    // the threshold compares the binary32 message, 4n bytes (= 2 * (2n) as BF16 elements)
    const lpar_codec_t eff = lpar_effective_codec(2 * n, codec, opts);
    if (workspace_bytes < lpar_collective_workspace_bytes(LPAR_OP_ALLREDUCE_F32, N, n, eff))
        return LPAR_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (opts && opts->stage_events[0]) cudaEventRecord(opts->stage_events[0], stream);
    if (eff == LPAR_CODEC_BF16) {
        launch_f32_reduce(in, N, reinterpret_cast<float *>(ws), o, 4 * n / 16, stream);
    } else {
        const size_t wb = lpar_wire_bytes(eff, n);
        OutPtrs wires{};
        for (int r = 0; r < N; ++r) wires.p[r] = ws + (size_t)r * wb;
        bool ok = false;
        switch (eff) {
        case LPAR_CODEC_INT4: ok = launch_f32_c<kINT4>(in, wires, N, ws + (size_t)N * wb, o, n / kTileElems, stream); break;
        case LPAR_CODEC_INT3: ok = launch_f32_c<kINT3>(in, wires, N, ws + (size_t)N * wb, o, n / kTileElems, stream); break;
        case LPAR_CODEC_FP8_E4M3: ok = launch_f32_c<kFP8>(in, wires, N, ws + (size_t)N * wb, o, n / kTileElems, stream); break;
        case LPAR_CODEC_MXFP4: ok = launch_f32_c<kMXFP4>(in, wires, N, ws + (size_t)N * wb, o, n / kTileElems, stream); break;
        default: break;
        }
        if (!ok) return LPAR_ERR_CUDA;
    }
    if (opts && opts->stage_events[1]) cudaEventRecord(opts->stage_events[1], stream);
    return launch_status();
}
