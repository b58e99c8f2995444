// lpar_static_ws.cu -- lpar_allreduce_static: the all-reduce with a workspace
// that lives inside the library, for callers that cannot allocate device
// memory themselves.
//
// Who needs it: code that runs where device allocation is not available or not
// allowed -- for example a plugin or extension whose host application owns all
// device memory and exposes no allocator to it, or a serving loop that runs
// under a fixed memory budget and must not grow its footprint (or pay for an
// allocation) on the communication path.  Such callers still own and pass
// their input and output buffers; only the scratch space is provided here.
//
// The scratch is one file-scope __device__ array of LPAR_STATIC_WORKSPACE_BYTES.
// A GPU holds it from the moment the library's module is loaded there (with
// CUDA's lazy module loading, no later than the first call on that device)
// until the process exits.  Host code cannot use the array's name as a device
// address, so a call looks the address up with cudaGetSymbolAddress (with the
// device current) the first time it runs in a given device context, caches
// it together with that context, and looks it up again whenever the current
// context differs (another context on the device, or a fresh primary context
// after cudaDeviceReset); make the first call before any stream capture.  All
// calls share the array and it keeps the last call's contents: nothing in it
// needs to start at zero (every byte the all-reduce reads there it has written
// first in the same call), but calls whose work overlaps on the GPU -- on
// different streams, or on different host threads without ordering -- race on
// it and must be serialised by the caller.
#include "lpar.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[LPAR_STATIC_WORKSPACE_BYTES];

// The current CUDA context, through the driver entry point the runtime hands
// out (the library does not link the driver library itself); null when it
// cannot be had.
CUcontext current_context() {
    using Fn = CUresult (*)(CUcontext *);
    static Fn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<Fn>(nullptr);
        return reinterpret_cast<Fn>(f);
    }();
    CUcontext ctx = nullptr;
    if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

struct Cached {
    std::mutex lock;
    CUcontext ctx = nullptr;
    void *addr = nullptr;
};

// Device address of g_static_workspace in the current device context (cached
// per device, together with the context it belongs to).
lpar_status_t static_workspace(void **ptr) {
    static Cached cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LPAR_ERR_CUDA;
    Cached &c = cache[dev];
    std::lock_guard<std::mutex> held(c.lock);
    CUcontext ctx = current_context();
    if (!c.addr || !ctx || ctx != c.ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return LPAR_ERR_CUDA;
        // the lookup makes the device's primary context current if none was
        ctx = current_context();
        c.addr = p;
        c.ctx = ctx;
    }
    *ptr = c.addr;
    return LPAR_OK;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) lpar_status_t
lpar_allreduce_static(const void *const *inputs, int N, size_t n, lpar_codec_t codec, void *const *out,
                      const lpar_options_t *opts, cudaStream_t stream) {
    const size_t need = lpar_workspace_bytes(N, n, lpar_effective_codec(n, codec, opts));
    if (need > LPAR_STATIC_WORKSPACE_BYTES) return LPAR_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    const lpar_status_t st = static_workspace(&ws);
    if (st != LPAR_OK) return st;
    return lpar_allreduce(inputs, N, n, codec, out, ws, LPAR_STATIC_WORKSPACE_BYTES, opts, stream);
}
