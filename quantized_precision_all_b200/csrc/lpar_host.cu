// lpar_host.cu -- lpar_allreduce_host and lpar_allreduce_f32_host: the
// all-reduce of BF16 or binary32 messages held in host memory, with the copies
// in both directions and the kernels overlapped.
//
// A tile's result depends only on the same tile of every rank, so the message
// can be reduced chunk by chunk (chunks of whole tiles) and the result is the
// one a single lpar_allreduce of the whole message gives.  Three streams carry
// the work of chunk k, in a ring of three device staging slots (slot k % 3,
// each holding the N ranks' chunk, reduced in place):
//   up    waits until slot k % 3 has been copied out (chunk k - 3), copies the
//         N input chunks in;
//   comp  waits for them, runs lpar_allreduce (lpar_allreduce_f32) in place;
//   down  waits for it, copies the N result chunks out.
// So the upload of chunk k + 1, the kernel of chunk k and the download of
// chunk k - 1 run at the same time: with page-locked host buffers the time is
// bound by the slower PCIe direction instead of the sum of both.  The
// threshold is decided once, on the whole message, and every chunk runs with
// the codec it selects.  The three streams and their events are created on a
// device's first call and kept for the life of the process (one set per
// device, in the device's primary context); a per-device lock makes each
// call's enqueue complete before another thread's begins, so concurrent
// callers never interleave their event records.  Every call starts after
// the work already on the caller's stream and ends by making that stream wait
// for all of its own work.
#include "lpar.h"

#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>
#include <nvtx3/nvToolsExt.h>

#define LPAR_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kTile = 2048;   // elements per tile
constexpr int kSlots = 3;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around the call (host-side enqueue), as for every C ABI call.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

size_t round16(size_t b) { return (b + 15) & ~(size_t)15; }

// Byte layout of the device buffer: kSlots x N chunk buffers (bytes per
// element x chunk each, 16-byte aligned), then the workspace of one chunk.

struct Pipeline {
    cudaStream_t st[3] = {nullptr, nullptr, nullptr};   // up, comp, down
    cudaEvent_t start = nullptr, up[kSlots] = {}, comp[kSlots] = {}, down[kSlots] = {};
    bool ok = true;

    Pipeline() {
        for (auto &s : st) ok = ok && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess;
        for (int k = 0; k < kSlots; ++k) {
            ok = ok && cudaEventCreateWithFlags(&up[k], cudaEventDisableTiming) == cudaSuccess;
            ok = ok && cudaEventCreateWithFlags(&comp[k], cudaEventDisableTiming) == cudaSuccess;
            ok = ok && cudaEventCreateWithFlags(&down[k], cudaEventDisableTiming) == cudaSuccess;
        }
    }
};

constexpr int kMaxDevices = 64;

// The current device's pipeline and its lock; created on first use and never
// destroyed (the process's exit releases them).  Null when the device cannot
// be queried or the streams cannot be created.
struct DevicePipeline {
    std::mutex lock;
    Pipeline *p = nullptr;
};

DevicePipeline *device_pipeline() {
    static DevicePipeline per_device[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    return &per_device[dev];
}

// Device bytes of the pipeline: three slots of N chunks of `elem` bytes per
// element, then the workspace `ws` of one chunk.
size_t staging_bytes(int N, size_t chunk, size_t elem, size_t ws) {
    return (size_t)kSlots * N * round16(elem * chunk) + round16(ws);
}

// The pipeline of lpar_allreduce_host / lpar_allreduce_f32_host: `elem` bytes
// per element, `ws_need(chunk)` the workspace of one chunk, `reduce` the
// in-place all-reduce of one chunk on a stream.
template <class WsNeed, class Reduce>
lpar_status_t host_pipeline(const void *const *host_inputs, int N, size_t n, void *const *host_out, size_t chunk,
                            void *device, size_t device_bytes, size_t elem, WsNeed ws_need, Reduce reduce,
                            const lpar_options_t *opts, cudaStream_t stream) {
    if (chunk > n) chunk = n;
    if (device_bytes < staging_bytes(N, chunk, elem, ws_need(chunk))) return LPAR_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *const base = static_cast<uint8_t *>(device);
    const size_t cb = round16(elem * chunk);
    uint8_t *const ws = base + (size_t)kSlots * N * cb;
    const size_t ws_bytes = device_bytes - (size_t)kSlots * N * cb;

    DevicePipeline *dp = device_pipeline();
    if (!dp) return LPAR_ERR_CUDA;
    std::lock_guard<std::mutex> held(dp->lock);
    if (!dp->p) {
        Pipeline *fresh = new Pipeline();
        if (!fresh->ok) return LPAR_ERR_CUDA;      // a failed set is dropped, not released
        dp->p = fresh;
    }
    Pipeline &p = *dp->p;
    cudaStream_t up = p.st[0], comp = p.st[1], down = p.st[2];
    if (opts && opts->stage_events[0]) cudaEventRecord(opts->stage_events[0], stream);
    if (cudaEventRecord(p.start, stream) != cudaSuccess) return LPAR_ERR_CUDA;
    for (cudaStream_t s : p.st)
        if (cudaStreamWaitEvent(s, p.start, 0) != cudaSuccess) return LPAR_ERR_CUDA;

    const size_t chunks = (n + chunk - 1) / chunk;
    lpar_status_t status = LPAR_OK;
    for (size_t k = 0; k < chunks && status == LPAR_OK; ++k) {
        const int s = (int)(k % kSlots);
        const size_t e0 = k * chunk, elems = (n - e0 < chunk) ? n - e0 : chunk;
        const void *in[LPAR_MAX_RANKS];
        void *out[LPAR_MAX_RANKS];
        for (int r = 0; r < N; ++r) {
            uint8_t *slot = base + ((size_t)s * N + r) * cb;
            in[r] = slot;
            out[r] = slot;
        }
        bool ok = true;
        // up: the slot is free once chunk k - 3 has been copied out
        if (k >= kSlots) ok = ok && cudaStreamWaitEvent(up, p.down[s], 0) == cudaSuccess;
        for (int r = 0; r < N && ok; ++r)
            ok = cudaMemcpyAsync(out[r], static_cast<const uint8_t *>(host_inputs[r]) + elem * e0, elem * elems,
                                 cudaMemcpyHostToDevice, up) == cudaSuccess;
        ok = ok && cudaEventRecord(p.up[s], up) == cudaSuccess;
        // comp: the all-reduce of the chunk, in place
        ok = ok && cudaStreamWaitEvent(comp, p.up[s], 0) == cudaSuccess;
        if (!ok) { status = LPAR_ERR_CUDA; break; }
        status = reduce(in, elems, out, ws, ws_bytes, comp);
        if (status != LPAR_OK) break;
        ok = cudaEventRecord(p.comp[s], comp) == cudaSuccess;
        // down: the N result chunks back to the host
        ok = ok && cudaStreamWaitEvent(down, p.comp[s], 0) == cudaSuccess;
        for (int r = 0; r < N && ok; ++r)
            ok = cudaMemcpyAsync(static_cast<uint8_t *>(host_out[r]) + elem * e0, out[r], elem * elems,
                                 cudaMemcpyDeviceToHost, down) == cudaSuccess;
        ok = ok && cudaEventRecord(p.down[s], down) == cudaSuccess;
        if (!ok) status = LPAR_ERR_CUDA;
    }
    // Later work on `stream` runs after everything enqueued here, also after an
    // error, so that the caller may release the staging and host buffers once
    // `stream` has passed this point.
    for (int i = 0; i < 3; ++i) {
        cudaEvent_t done = i == 0 ? p.up[0] : (i == 1 ? p.comp[0] : p.down[0]);
        if (cudaEventRecord(done, p.st[i]) != cudaSuccess || cudaStreamWaitEvent(stream, done, 0) != cudaSuccess)
            status = LPAR_ERR_CUDA;
    }
    if (status != LPAR_OK) return status;
    if (opts && opts->stage_events[1]) cudaEventRecord(opts->stage_events[1], stream);
    return cudaGetLastError() == cudaSuccess ? LPAR_OK : LPAR_ERR_CUDA;
}

// Argument checks shared by both entry points (before anything is enqueued).
lpar_status_t check_host_args(const void *const *host_inputs, int N, size_t n, lpar_codec_t codec,
                              void *const *host_out, size_t chunk, const void *device, const lpar_options_t *opts) {
    if (N < 1 || N > LPAR_MAX_RANKS || n % kTile || chunk == 0 || chunk % kTile) return LPAR_ERR_INVALID_ARG;
    if (codec < LPAR_CODEC_BF16 || codec > LPAR_CODEC_MXFP4) return LPAR_ERR_UNSUPPORTED;
    if (opts && opts->schedule > LPAR_SCHEDULE_ONE_SHOT) return LPAR_ERR_UNSUPPORTED;
    if (n == 0) return LPAR_OK;
    if (!host_inputs || !host_out || !device) return LPAR_ERR_INVALID_ARG;
    for (int r = 0; r < N; ++r)
        if (!host_inputs[r] || !host_out[r]) return LPAR_ERR_INVALID_ARG;
    if (!aligned16(device)) return LPAR_ERR_MISALIGNED;
    return LPAR_OK;
}

}  // namespace

LPAR_API size_t lpar_host_staging_bytes(int N, size_t chunk, lpar_codec_t codec) {
    if (N < 1 || N > LPAR_MAX_RANKS || chunk == 0 || chunk % kTile) return 0;
    const size_t ws = lpar_workspace_bytes(N, chunk, codec);
    if (ws == 0 && codec != LPAR_CODEC_BF16) return 0;
    return staging_bytes(N, chunk, 2, ws);
}

LPAR_API size_t lpar_host_staging_bytes_f32(int N, size_t chunk, lpar_codec_t codec) {
    if (N < 1 || N > LPAR_MAX_RANKS || chunk == 0 || chunk % kTile) return 0;
    const size_t ws = lpar_collective_workspace_bytes(LPAR_OP_ALLREDUCE_F32, N, chunk, codec);
    if (ws == 0) return 0;
    return staging_bytes(N, chunk, 4, ws);
}

LPAR_API lpar_status_t lpar_allreduce_host(const void *const *host_inputs, int N, size_t n, lpar_codec_t codec,
                                           void *const *host_out, size_t chunk, void *device, size_t device_bytes,
                                           const lpar_options_t *opts, cudaStream_t stream) {
    Range trace("lpar_allreduce_host");
    const lpar_status_t st = check_host_args(host_inputs, N, n, codec, host_out, chunk, device, opts);
    if (st != LPAR_OK || n == 0) return st;
    const lpar_codec_t eff = lpar_effective_codec(n, codec, opts);    // decided on the whole message
    lpar_options_t per_chunk{};
    per_chunk.schedule = opts ? opts->schedule : LPAR_SCHEDULE_AUTO;
    return host_pipeline(
        host_inputs, N, n, host_out, chunk, device, device_bytes, 2,
        [&](size_t c) { return lpar_workspace_bytes(N, c, eff); },
        [&](const void *const *in, size_t elems, void *const *out, void *ws, size_t wsb, cudaStream_t s) {
            return lpar_allreduce(in, N, elems, eff, out, ws, wsb, &per_chunk, s);
        },
        opts, stream);
}

LPAR_API lpar_status_t lpar_allreduce_f32_host(const void *const *host_inputs, int N, size_t n, lpar_codec_t codec,
                                               void *const *host_out, size_t chunk, void *device,
                                               size_t device_bytes, const lpar_options_t *opts, cudaStream_t stream) {
    Range trace("lpar_allreduce_f32_host");
    const lpar_status_t st = check_host_args(host_inputs, N, n, codec, host_out, chunk, device, opts);
    if (st != LPAR_OK || n == 0) return st;
    const int schedule = opts ? (int)opts->schedule : (int)LPAR_SCHEDULE_AUTO;
    if (schedule != LPAR_SCHEDULE_AUTO && schedule != LPAR_SCHEDULE_SINGLE_PASS) return LPAR_ERR_UNSUPPORTED;
    // the threshold compares the binary32 message, 4n bytes (= 2 * (2n) as BF16 elements)
    const lpar_codec_t eff = lpar_effective_codec(2 * n, codec, opts);
    lpar_options_t per_chunk{};
    per_chunk.schedule = (lpar_schedule_t)schedule;
    return host_pipeline(
        host_inputs, N, n, host_out, chunk, device, device_bytes, 4,
        [&](size_t c) { return lpar_collective_workspace_bytes(LPAR_OP_ALLREDUCE_F32, N, c, eff); },
        [&](const void *const *in, size_t elems, void *const *out, void *ws, size_t wsb, cudaStream_t s) {
            return lpar_allreduce_f32(in, N, elems, eff, out, ws, wsb, &per_chunk, s);
        },
        opts, stream);
}
