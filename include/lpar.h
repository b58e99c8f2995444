/*
 * lpar.h -- C ABI of the B200 (sm_100a) compressed all-reduce library.
 *
 * The library implements the two-shot low-precision all-reduce that these
 * pages describe, with N "ranks" whose buffers all sit in one GPU's HBM:
 *
 *   stage 1  quantise   every rank's BF16 message into a wire of tiles
 *   stage 2  reduce     per tile: dequantise the N wires, sum in FP32 in
 *                       ascending rank order, requantise with the same codec
 *                       (reduce-scatter receiver + all-gather producer)
 *   stage 3  decode     the gathered wire back to BF16, once per rank
 *
 * Sources, by page title and section:
 *  - "QuickReduce INT3 Quantization and Benchmarking on MI355": Summary (a
 *    transmitted tile is 1152 B with INT4 and 896 B with INT3), Method
 *    (block-level FP16 scale, symmetric codes, INT3 split into a low-2-bit
 *    plane "q2w" and a high-1-bit plane "q1w"), In practice (1 MB activation
 *    threshold for INT3).
 *  - "RCCLX: Innovating GPU communications on AMD platforms": Low-Precision
 *    Collectives (FP8 on the wire, computation in FP32), Direct Data Access
 *    (tree all-reduce = reduce-scatter followed by all-gather).
 *  - "FP8 Formats for Deep Learning", abstract (E4M3: no infinities, one NaN
 *    pattern, so 448 is the largest finite value).
 *  - "Microscaling Data Formats for Deep Learning", abstract (narrow
 *    floating-point elements sharing one per-block scale), with the INT3
 *    page's Summary naming the FP4 mode of the same all-reduce.
 *
 * Formats (readings where the pages are silent are marked "reading"):
 *  - A tile is 2048 consecutive elements made of 64 blocks of 32 (reading,
 *    the only split consistent with the printed tile sizes and FP16 scales).
 *  - INT4 tile (1152 B): 1024 B of 4-bit codes (element i in byte i/2, low
 *    nibble for even i), then 64 little-endian binary16 scales.
 *  - INT3 tile (896 B): q2w plane (512 B, element i's code & 3 at bits
 *    2*(i%4) of byte i/4), q1w plane (256 B, element i's code >> 2 at bit i%8
 *    of byte i/8), then 64 little-endian binary16 scales.
 *  - INT codes: s = f16_rne(fl32(absmax / qmax)) saturating at 65504,
 *    q = clamp(RNE(x / s), -qmax, qmax) of the exact quotient, stored as
 *    offset binary q + 2^(b-1); qmax = 7 (INT4) or 3 (INT3); s = 0 gives q = 0.
 *  - FP8 tile (2304 B): 2048 E4M3 codes, then 64 little-endian binary32 scales
 *    s = fl32(absmax / 448); a block with s < 2^-126 is stored as s = 0 and
 *    codes 0; otherwise code = e4m3_rne_satfinite(fl32(x * fl32(1 / s))).
 *  - MXFP4 tile (1088 B): 1024 B of E2M1 codes (element i in byte i/2, low
 *    nibble for even i; 1 sign, 2 exponent bits with bias 1, 1 mantissa bit:
 *    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), then 64 E8M0 scale bytes
 *    (value 2^(byte - 127)).  E = clamp(floor(log2(absmax)) - 2, -127, 127)
 *    (-127 for an all-zero block), code = e2m1_rne(x / 2^E) with magnitudes
 *    above 6 saturating to 6 and the sign kept (a negative value that rounds
 *    to zero gives code 0x8).
 *  - BF16 "tile" (4096 B): the BF16 values themselves (no compression).
 *  - Dequantised value: (float)q * s for INT (exact), fl32(e4m3(code) * s) for
 *    FP8, e2m1(code) * 2^E for MXFP4 (exact).  Final output: bf16_rne of the
 *    dequantised gathered value.
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers on the current CUDA device; the
 *    pointer ARRAYS (inputs, out, wires) are HOST arrays of N device pointers.
 *  - n is the number of BF16 elements per rank and must be a multiple of
 *    LPAR_TILE_ELEMS, at most 2^44; n == 0 is a valid no-op.  N must be in
 *    [1, LPAR_MAX_RANKS].
 *  - Every data pointer must be 16-byte aligned.
 *  - The caller owns all memory.  The library (lpar_peer_alloc and
 *    lpar_peer_free aside, whose job it is) allocates nothing, frees
 *    nothing, never synchronises and keeps no pointer after a call returns.
 *    Work is enqueued on `stream` asynchronously; buffers must stay valid
 *    until the stream has passed the call.
 *  - Argument errors are detected before anything is launched and return a
 *    status other than LPAR_OK.  A failed launch returns LPAR_ERR_CUDA.
 *    Faults during execution surface at the caller's next synchronisation.
 *    No call aborts, exits or throws.
 */
#ifndef LPAR_H
#define LPAR_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LPAR_TILE_ELEMS 2048
#define LPAR_BLOCK_ELEMS 32
#define LPAR_MAX_RANKS 8

typedef enum {
    LPAR_CODEC_BF16 = 0,      /* uncompressed passthrough, 4096 B per tile */
    LPAR_CODEC_FP8_E4M3 = 1,  /* E4M3 codes + binary32 scale per 32 elements, 2304 B per tile */
    LPAR_CODEC_INT4 = 2,      /* 4-bit codes + binary16 scale per 32 elements, 1152 B per tile */
    LPAR_CODEC_INT3 = 3,      /* q2w + q1w planes + binary16 scale per 32, 896 B per tile */
    LPAR_CODEC_MXFP4 = 4      /* E2M1 codes + E8M0 (power of two) scale per 32, 1088 B per tile */
} lpar_codec_t;

typedef enum {
    LPAR_OK = 0,
    LPAR_ERR_INVALID_ARG = 1,          /* null pointer, N or n out of range, bad tile range */
    LPAR_ERR_MISALIGNED = 2,           /* a data pointer is not 16-byte aligned */
    LPAR_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < lpar_workspace_bytes(...) */
    LPAR_ERR_UNSUPPORTED = 4,          /* unknown codec or schedule */
    LPAR_ERR_CUDA = 5                  /* a CUDA launch or device query failed */
} lpar_status_t;

typedef enum {
    LPAR_SCHEDULE_AUTO = 0,        /* the library's choice (currently LPAR_SCHEDULE_SINGLE_PASS) */
    LPAR_SCHEDULE_FUSED = 1,       /* quantise; reduce + requantise + decode in one kernel */
    LPAR_SCHEDULE_THREE_STAGE = 2, /* quantise; reduce + requantise; decode (three kernels) */
    LPAR_SCHEDULE_SINGLE_PASS = 3, /* one kernel: each CTA quantises a chunk of every rank, then
                                      reduces, requantises and decodes that chunk from the wires
                                      it has just written (same results, one launch) */
    LPAR_SCHEDULE_ONE_SHOT = 4     /* a different algorithm, the one-shot ("flat") all-reduce of the
                                      RCCLX page's Direct Data Access section: every rank reduces
                                      all N stage-1 wires itself and rounds the FP32 sum once to
                                      BF16, with no requantisation.  One quantisation stage instead
                                      of two, so its results differ from the schedules above (they
                                      equal lpar_reduce_scatter's, gathered). */
} lpar_schedule_t;

typedef enum {
    LPAR_OP_ALLREDUCE = 0,
    LPAR_OP_REDUCE_SCATTER = 1,
    LPAR_OP_ALL_GATHER = 2,
    LPAR_OP_ALL_TO_ALL = 3,
    LPAR_OP_ALLREDUCE_F32 = 4
} lpar_collective_t;

typedef struct {
    /* A quantising codec runs only when the per-rank message (2*n bytes) is at
     * least this many bytes; smaller messages take the BF16 passthrough.
     * 0 = always quantise.  The INT3 page recommends 1 MB (1 << 20). */
    size_t min_quant_bytes;
    lpar_schedule_t schedule;      /* 0 (LPAR_SCHEDULE_AUTO) is the default */
    /* Optional tracing: events recorded on `stream` at the stage boundaries --
     * [0] before stage 1, [1] after stage 1, [2] after stage 2 (after the
     * fused reduce+decode in the fused schedule), [3] after stage 3 (three-
     * stage schedule only).  The single-pass schedule records [0] before and
     * [1] after its one kernel.  NULL entries are skipped.  The BF16
     * passthrough has no stage 1: [0] and [1] are recorded back to back, then
     * [2] after its (fused, or single-pass) kernel. */
    cudaEvent_t stage_events[4];
} lpar_options_t;

/* Bytes of one 2048-element tile: 4096 (BF16), 2304 (FP8), 1152 (INT4), 896
 * (INT3), 1088 (MXFP4); 0 for an unknown codec. */
size_t lpar_tile_bytes(lpar_codec_t codec);

/* Bytes of the wire of an n-element message: (n / 2048) * lpar_tile_bytes(codec). */
size_t lpar_wire_bytes(lpar_codec_t codec, size_t n);

/* Workspace lpar_allreduce needs when it runs `codec`: N stage-1 wires plus one
 * gathered wire for a quantising codec, one gathered wire (2n bytes) for BF16;
 * 0 for N outside [1, LPAR_MAX_RANKS] or an unknown codec.  With a threshold
 * set, size it for lpar_effective_codec(n, codec, opts). */
size_t lpar_workspace_bytes(int N, size_t n, lpar_codec_t codec);

/* Stage 1 for one rank: in_bf16 (n BF16 values) -> wire
 * (lpar_wire_bytes(codec, n) bytes).  For BF16 the wire is a copy. */
lpar_status_t lpar_quantize(const void *in_bf16, size_t n, lpar_codec_t codec,
                            void *wire, cudaStream_t stream);

/* Stage 2 for the tiles [tile_begin, tile_begin + tile_count) of N full
 * wires: wires[r] is the base of rank r's wire; tile t of every wire is
 * dequantised, summed in FP32 in ascending rank order starting from +0.0f,
 * requantised, and written as tile t of wire_out (the base of the gathered
 * wire).  wire_out must not overlap any wires[r]. */
lpar_status_t lpar_reduce(const void *const *wires, int N, size_t tile_begin, size_t tile_count,
                          lpar_codec_t codec, void *wire_out, cudaStream_t stream);

/* Stage 3: wire (n elements' worth) -> out_bf16 (n BF16 values, RNE). */
lpar_status_t lpar_decode(const void *wire, size_t n, lpar_codec_t codec,
                          void *out_bf16, cudaStream_t stream);

/* The whole all-reduce of N ranks' BF16 messages of n elements: inputs[r] ->
 * every out[r] receives the same BF16 result.  out[r] may equal inputs[r]
 * (in place); out buffers must not overlap each other or the workspace.
 * workspace: device memory of at least lpar_workspace_bytes(N, n, effective
 * codec) bytes, 16-byte aligned, contents ignored and overwritten.
 * opts may be NULL (always quantise, LPAR_SCHEDULE_AUTO).  Every schedule
 * gives the same bits, except LPAR_SCHEDULE_ONE_SHOT (a different algorithm,
 * see lpar_schedule_t), which needs only N wires of the workspace. */
lpar_status_t lpar_allreduce(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                             void *const *out, void *workspace, size_t workspace_bytes,
                             const lpar_options_t *opts, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Standalone low-precision collectives (the RCCLX page's Low-Precision
 * Collectives section: the quantised wire serves the other collectives too).
 * Each rank's message is quantised once (stage 1) into a wire in the
 * workspace; the receiver works from the wire.  No second quantisation: a
 * reduction rounds its FP32 sum (ascending rank order from +0.0f) once to
 * BF16.  Conventions as for lpar_allreduce (device buffers 16-byte aligned,
 * host pointer arrays, asynchronous on `stream`, argument errors before any
 * launch); outputs must not overlap the inputs, each other or the workspace.
 * opts->min_quant_bytes applies to the per-rank message named below (smaller
 * messages move the BF16 values themselves); opts->schedule is ignored;
 * opts->stage_events[0] and [1] are recorded before and after the one kernel.
 * ------------------------------------------------------------------------- */

/* Workspace bytes of a collective for the codec that runs (after the
 * threshold): the all-reduce as lpar_workspace_bytes(N, size, codec); the
 * all-reduce of binary32 messages (N + 1) wires, or 4 * size bytes for the
 * uncompressed passthrough; the others N wires of their per-rank message
 * (reduce-scatter: n elements; all-gather: m; all-to-all: N * m), and 0 for
 * BF16, when no workspace is needed and `workspace` may be NULL.  `size` is
 * each call's size argument.  0 for N outside [1, LPAR_MAX_RANKS] or an
 * unknown codec or op. */
size_t lpar_collective_workspace_bytes(lpar_collective_t op, int N, size_t size, lpar_codec_t codec);

/* Reduce-scatter of N BF16 messages of n elements (n a multiple of 2048): the
 * T = n / 2048 tiles are split into N shards by the floor partition, shard j =
 * tiles [j*T/N, (j+1)*T/N), and out[j] receives shard j of the BF16 sum from
 * element 0 (so out[j] holds (floor((j+1)T/N) - floor(jT/N)) * 2048 values;
 * an empty shard writes nothing).  Threshold on 2n bytes. */
lpar_status_t lpar_reduce_scatter(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                  void *const *out, void *workspace, size_t workspace_bytes,
                                  const lpar_options_t *opts, cudaStream_t stream);

/* All-gather: rank r contributes m elements (m a multiple of 2048); every
 * out[j] (N * m values) receives rank r's contribution, decoded from rank r's
 * wire, at elements [r*m, (r+1)*m).  Threshold on 2m bytes. */
lpar_status_t lpar_all_gather(const void *const *inputs, int N, size_t m, lpar_codec_t codec,
                              void *const *out, void *workspace, size_t workspace_bytes,
                              const lpar_options_t *opts, cudaStream_t stream);

/* All-to-all: inputs[r] holds N segments of m elements (m a multiple of 2048),
 * segment j bound for rank j; out[j] (N * m values) receives rank r's segment
 * j, decoded from rank r's wire, at elements [r*m, (r+1)*m).  Threshold on
 * the whole per-rank message, 2*N*m bytes. */
lpar_status_t lpar_all_to_all(const void *const *inputs, int N, size_t m, lpar_codec_t codec,
                              void *const *out, void *workspace, size_t workspace_bytes,
                              const lpar_options_t *opts, cudaStream_t stream);

/* The all-reduce of N binary32 messages of n elements (the RCCLX page's
 * Low-Precision Collectives: FP32 or BF16 inputs, FP8 for up to 4:1 against
 * FP32).  Same codecs, tiles and stages as lpar_allreduce; each out[r] (n
 * binary32 values) receives the dequantised gathered value itself, with no
 * rounding to BF16.  LPAR_CODEC_BF16 selects the uncompressed passthrough:
 * the binary32 sum in ascending rank order from +0.0f.  The threshold
 * compares the binary32 message, 4n bytes.  Workspace:
 * lpar_collective_workspace_bytes(LPAR_OP_ALLREDUCE_F32, N, n, effective
 * codec).  Schedules: LPAR_SCHEDULE_AUTO and LPAR_SCHEDULE_SINGLE_PASS (one
 * kernel); others return LPAR_ERR_UNSUPPORTED.  In place (out[r] ==
 * inputs[r]) is allowed.  Stage events [0] and [1] bracket the kernel. */
lpar_status_t lpar_allreduce_f32(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                 void *const *out, void *workspace, size_t workspace_bytes,
                                 const lpar_options_t *opts, cudaStream_t stream);

/* Size of the workspace that lpar_allreduce_static keeps inside the library. */
#define LPAR_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)

/* lpar_allreduce without a caller-provided workspace, for callers that cannot
 * allocate device memory (for example a plugin whose host application owns all
 * device memory, or a loop held to a fixed memory budget).  The pages have no
 * counterpart: this is a deployment convenience, not part of the method.
 * Inputs, outputs, options and stream are as for lpar_allreduce; the workspace
 * is a 16 MiB array inside the library, reserved on a device when the
 * library's code is loaded there (with CUDA's lazy module loading, no later
 * than the first call on that device) and held until the process exits.
 * Returns LPAR_ERR_WORKSPACE_TOO_SMALL when lpar_workspace_bytes(N, n,
 * effective codec) exceeds LPAR_STATIC_WORKSPACE_BYTES (e.g. INT3 with N = 2
 * up to n = 12.8 Mi), and never calls cudaMalloc/cudaFree.  The first call in
 * a device context looks up the array's device address (cudaGetSymbolAddress)
 * and caches it with that context; a call in another context (another context
 * on the device, or the new primary context after cudaDeviceReset) looks it up
 * again.  Make the first call before any stream capture.  All calls share the
 * one array: calls whose work overlaps on the GPU race on it and must be
 * serialised by the caller. */
lpar_status_t lpar_allreduce_static(const void *const *inputs, int N, size_t n, lpar_codec_t codec,
                                    void *const *out, const lpar_options_t *opts, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The all-reduce of messages held in host memory.  The pages have no
 * counterpart; it serves callers whose tensors live on the host.  A tile's
 * result depends only on the same tile of every rank, so the message is
 * reduced chunk by chunk (chunks of whole tiles) on three streams of the
 * library's own -- upload of chunk k + 1, lpar_allreduce of chunk k (in place,
 * in device staging) and download of chunk k - 1 at the same time -- and the
 * result equals that of one lpar_allreduce of the whole message with the same
 * options.  The threshold opts->min_quant_bytes is decided once on the whole
 * message (2n bytes); opts->schedule applies to every chunk; stage events [0]
 * and [1] are recorded on `stream` before the first copy and after the last.
 * ------------------------------------------------------------------------- */

/* Device bytes lpar_allreduce_host needs for chunks of `chunk` elements (a
 * multiple of 2048) with `codec` (the one that runs after the threshold):
 * three staging slots of N chunks plus the workspace of one chunk.  0 for N
 * outside [1, LPAR_MAX_RANKS], chunk 0 or not a multiple of 2048, or an
 * unknown codec. */
size_t lpar_host_staging_bytes(int N, size_t chunk, lpar_codec_t codec);

/* host_inputs[r], host_out[r]: N host arrays of n BF16 values (n a multiple of
 * 2048); host_out[r] may equal host_inputs[r].  Page-locked host memory
 * (cudaHostAlloc or cudaHostRegister) lets the copies overlap each other and
 * the kernels; pageable memory gives the same result with the copies
 * serialised.  chunk: elements per chunk, a multiple of 2048 (a chunk larger
 * than n is n).  device: at least lpar_host_staging_bytes(N, min(chunk, n),
 * effective codec) bytes of device memory, 16-byte aligned, owned by the
 * caller.  The work is ordered after earlier work on `stream`, and later work
 * on `stream` runs after the last result has reached host memory; the call
 * returns once everything is enqueued.  The copies and kernels run on three
 * streams of the library's own, created on a device's first call (in the
 * current context, normally the primary one) and kept until the process
 * exits; calls from several host threads are serialised while they enqueue.
 * Not for stream capture.  Argument errors are
 * returned before anything is enqueued; after an error returned once copies
 * or kernels were enqueued, later work on `stream` still runs after them, so
 * the buffers may be released once `stream` has passed the call. */
lpar_status_t lpar_allreduce_host(const void *const *host_inputs, int N, size_t n, lpar_codec_t codec,
                                  void *const *host_out, size_t chunk, void *device, size_t device_bytes,
                                  const lpar_options_t *opts, cudaStream_t stream);

/* The same for binary32 messages: lpar_allreduce_f32 chunk by chunk.  Staging:
 * lpar_host_staging_bytes_f32(N, min(chunk, n), effective codec), the
 * threshold deciding on the binary32 message (4n bytes) as in
 * lpar_allreduce_f32; schedules LPAR_SCHEDULE_AUTO and
 * LPAR_SCHEDULE_SINGLE_PASS; otherwise as lpar_allreduce_host. */
size_t lpar_host_staging_bytes_f32(int N, size_t chunk, lpar_codec_t codec);
lpar_status_t lpar_allreduce_f32_host(const void *const *host_inputs, int N, size_t n, lpar_codec_t codec,
                                      void *const *host_out, size_t chunk, void *device, size_t device_bytes,
                                      const lpar_options_t *opts, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The all-reduce as one kernel per rank over peer memory ("RCCLX: Innovating
 * GPU communications on AMD platforms", Direct Data Access: ranks store into
 * each other's memory directly, and the tree all-reduce is a reduce-scatter
 * followed by an all-gather; Low-Precision Collectives: the quantised wire is
 * what crosses the links).  Each rank's launch quantises its message and
 * stores every wire tile straight into the mailbox of the tile's shard owner
 * (shard j = tiles [jT/N, (j+1)T/N) of the T tiles), reduces and requantises
 * its own shard once every rank's tiles have arrived and stores the reduced
 * tiles into every rank's gathered wire, then decodes the gathered wire into
 * its output.  Arrival is signalled by flag words that carry the call's epoch.
 * The results equal lpar_allreduce's (same codec, schedule irrelevant) bit for
 * bit.
 *
 * Per rank r, in memory the other ranks can reach (peer memory of another GPU
 * opened with lpar_peer_import, or, when all ranks run in one launch, plain
 * device memory):
 *   mailboxes[r]  lpar_peer_mailbox_bytes(N, n, codec) bytes
 *   gathered[r]   lpar_peer_gather_bytes(n, codec) bytes
 *   flags[r]      lpar_peer_flag_bytes(N, n) bytes, all zero before the first
 *                 call (lpar_peer_alloc zeroes) and left alone between calls
 * and, for the ranks this launch runs only, inputs[r] / outputs[r] (n BF16
 * values each, device memory of this GPU; an output may equal its input, as
 * each output tile is written only after every launch has read that tile).
 * All are host arrays of N pointers valid in the calling process, every
 * pointer 16-byte aligned.
 *
 * The launch runs ranks [rank0, rank0 + ranks).  With ranks == N it is the
 * whole all-reduce on this GPU (mailboxes and gathered wires in its HBM).
 * With ranks < N the other ranks must be running their own launches on other
 * GPUs (their buffers are memory of another device, or mapped host memory);
 * a rank outside the launch whose buffers are memory of the current device is
 * refused with LPAR_ERR_INVALID_ARG, because two launches on one GPU that
 * wait on each other are not guaranteed to run at the same time, and so is
 * one whose buffers are host memory the GPU cannot reach (not page-locked).
 *
 * timeout_ns (> 0): a wait for another rank's tiles gives up when it has seen
 * no arrival for this long (or after timeout_ns / 128 polls).
 * status: LPAR_PEER_STATUS_WORDS uint32 words of this GPU's memory, 16-byte
 * aligned, zero before the first call on a set of buffers and then left to
 * the kernel (one status per set of buffers and launching rank).  Word [4] is
 * the epoch of the last call: each launch reads it, uses one more as its own
 * epoch (the value its flags carry) and stores that when its last CTA
 * finishes, so calls captured in a CUDA graph stay correct on every replay;
 * every rank must make the same calls on its buffers in the same order.  [5]
 * counts finished CTAs during a launch.  A wait that gives up writes [0] = 1,
 * [1] = the phase (1: waiting for mailbox tiles, 2: waiting for gathered
 * tiles), [2] = the waiting rank, [3] = the flag's index, and every other wait
 * of the launch then stops too: the call ends with the outputs incomplete
 * instead of hanging.  A launch that finds [0] != 0 does nothing (it still
 * advances [4]).  After a failure the flags are in an unknown state: zero the
 * flags and the status words on every rank before the next call.
 *
 * The kernel is a cooperative launch (all its CTAs resident at once) on
 * `stream`.  Argument errors return before the launch; LPAR_ERR_UNSUPPORTED
 * for an unknown codec or a device without cooperative launch.
 * ------------------------------------------------------------------------- */
#define LPAR_PEER_STATUS_WORDS 8
#define LPAR_PEER_HANDLE_BYTES 64

/* Buffer sizes of lpar_allreduce_peer; 0 for N outside [1, LPAR_MAX_RANKS], an
 * unknown codec, n not a multiple of 2048 or above 2^44, and for n == 0. */
size_t lpar_peer_mailbox_bytes(int N, size_t n, lpar_codec_t codec);
size_t lpar_peer_gather_bytes(size_t n, lpar_codec_t codec);
size_t lpar_peer_flag_bytes(int N, size_t n);

lpar_status_t lpar_allreduce_peer(const void *const *inputs, void *const *outputs, void *const *mailboxes,
                                  void *const *gathered, void *const *flags, int N, int rank0, int ranks,
                                  size_t n, lpar_codec_t codec, uint64_t timeout_ns, uint32_t *status,
                                  cudaStream_t stream);

/* Buffers shared between processes (CUDA IPC), the one place the library
 * allocates: lpar_peer_alloc reserves `bytes` of device memory on the current
 * device, zeroes it and synchronises the device; lpar_peer_free releases it.
 * lpar_peer_export writes the LPAR_PEER_HANDLE_BYTES-byte handle of an
 * lpar_peer_alloc'd pointer; another process passes the handle to
 * lpar_peer_import to map the memory (peer access enabled as needed) and
 * unmaps it with lpar_peer_close.  A process cannot import its own handle.
 * LPAR_ERR_INVALID_ARG for a null argument, LPAR_ERR_CUDA when the CUDA call
 * fails. */
lpar_status_t lpar_peer_alloc(size_t bytes, void **ptr);
lpar_status_t lpar_peer_free(void *ptr);
lpar_status_t lpar_peer_export(const void *ptr, unsigned char *handle);
lpar_status_t lpar_peer_import(const unsigned char *handle, void **ptr);
lpar_status_t lpar_peer_close(void *ptr);

/* The codec lpar_allreduce runs for these arguments after the threshold. */
lpar_codec_t lpar_effective_codec(size_t n, lpar_codec_t codec, const lpar_options_t *opts);

/* A static, human-readable name of a status code. */
const char *lpar_status_string(lpar_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* LPAR_H */
