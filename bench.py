"""Benchmark of the compressed all-reduce on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--schedule fused|three_stage]
    python bench.py --sweep | --collectives | --floor       (one JSON line per point)

A step is one pass of the whole path (quantise -> reduce + requantise ->
decode, all ranks) for every codec of the workload, back to back.  Default
workload: ``large_int3_int4`` (2 ranks x 1 GiB BF16 per rank, INT3 then INT4),
the large-message configuration on which the HBM roofline target is defined;
its inputs (2 GiB) are far larger than the 126 MB L2, so no flush is needed
between steps.

Metric: GB/s = (ranks x per-rank BF16 bytes x codecs) / time.  On one GPU the
ranks are simulated in its HBM (the emulated reduce-scatter / all-gather) and
the roofline is the fraction of measured HBM bandwidth the dominant kernel
reaches.  With ``--gpus G > 1`` (torchrun, one process per GPU) the ranks are
the G processes: every GPU holds one rank's message of the workload's size and
the step is the real all-reduce across them (``distributed.DistributedAllreduce``:
the library's stage kernels, NCCL all-to-all and all-gather of the wire bytes);
its roofline is the NVLink bytes each rank sends.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "quantized all-reduce GB/s (N x input bytes/s) and % of HBM peak on 1 B200"
TILE = 2048
CODEC_C = {"bf16": 2.0, "fp8": 2304 / 2048, "int4": 1152 / 2048, "int3": 896 / 2048, "mxfp4": 1088 / 2048}
KERNEL_SOURCES = tuple("quantized_precision_all_b200/csrc/" + f for f in (
    "lpar_kernels.cu", "lpar_codec.cuh", "lpar_tiles.cuh", "lpar_collectives.cu", "lpar_f32.cu"))
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
REF_TILES_PER_STEP = 256            # reference arm: 0.5 Mi elements per rank per core per step
CPU_BASELINE_TILES = 16384          # cpu_baseline: 32 Mi elements (64 MiB) per rank
PAR_TILES_PER_CORE = 2048           # cpu_baseline on every core: 4 Mi elements per rank per core
HOST_CHUNK_BYTES = 32 << 20         # e2e: bytes of one chunk of the host all-reduce, all ranks together
ROTATE_BYTES = 512 << 20            # back-to-back timing: buffer sets rotated over at least this many bytes (4x L2)
NVLINK_GBS = 770.0                  # measured peer copy per direction per GPU on this machine's B200s


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def source_sha():
    """Hash of the kernel sources with comments and blank space removed, so that
    a measurement stays tied to the code it was taken on across comment edits."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy read+write)"
    return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


# ---- algorithmic bytes per launch (reads + writes the definition requires) ------
# The library's choice of the single-pass kernel form (lpar_kernels.cu,
# launch_single_cn): the rank-parallel tile form up to 256 tiles per rank (512
# for FP8); above, warp-local for INT3 with N <= 2 or below 512 MiB of input
# and for INT4 / MXFP4 below 128 MiB of input, CTA-wide otherwise and for FP8.
BULK_MIN_BYTES = 128 << 20
INT3_WARP_MAX_BYTES = 512 << 20


TILE_FORM_MAX_TILES = {"fp8": 512}           # others: 256


def single_pass_kernel(codec, N, n):
    in_bytes = N * 2 * n
    if n // TILE <= TILE_FORM_MAX_TILES.get(codec, 256):
        return "k_allreduce_tile<%s,N=%d>" % (codec, N)
    if codec == "fp8":
        warp = False
    elif codec == "int3":
        warp = N <= 2 or in_bytes < INT3_WARP_MAX_BYTES
    else:
        warp = in_bytes < BULK_MIN_BYTES
    return ("k_allreduce_single_warp<%s,N=%d>" if warp else "k_allreduce_single<%s,N=%d>") % (codec, N)


def kernel_names(codec, schedule, N, f32=False, n=None):
    if f32:
        return ["k_f32_reduce<N=%d>" % N] if codec == "bf16" else ["k_allreduce_single_f32<%s,N=%d>" % (codec, N)]
    if codec == "bf16":
        return ["k_bf16_reduce<N=%d,fused>" % N] if schedule != "three_stage" else \
            ["k_bf16_reduce<N=%d>" % N, "k_broadcast"]
    if schedule == "single_pass":
        return [single_pass_kernel(codec, N, n) if n is not None else "k_allreduce_single<%s,N=%d>" % (codec, N)]
    if schedule == "fused":
        return ["k_quantize<%s>" % codec, "k_reduce<%s,N=%d,fused>" % (codec, N)]
    return ["k_quantize<%s>" % codec, "k_reduce<%s,N=%d>" % (codec, N), "k_decode<%s>" % codec]


def algorithmic_bytes(kernel, codec, N, n):
    c = CODEC_C[codec]
    if kernel.startswith("k_allreduce_single_f32"):
        # N binary32 messages in, N wires out and back in, gathered wire out, N binary32 outputs out
        return N * n * (4 + c) + n * (N * c + c + 4 * N)
    if kernel.startswith("k_f32_reduce"):
        return n * (4 * N + 4 + 4 * N)
    if kernel.startswith("k_allreduce_single") or kernel.startswith("k_allreduce_tile"):
        # N BF16 messages in, N wires out and back in, gathered wire out, N outputs out
        return N * n * (2 + c) + n * (N * c + c + 2 * N)
    if kernel.startswith("k_quantize"):
        return N * n * (2 + c)                        # read N BF16 messages, write N wires
    if kernel.startswith("k_reduce") and kernel.endswith("fused>"):
        return n * (N * c + c + 2 * N)                # read N wires, write gathered wire + N outputs
    if kernel.startswith("k_reduce"):
        return n * (N * c + c)
    if kernel.startswith("k_decode"):
        return n * (c + 2 * N)
    if kernel.startswith("k_bf16_reduce") and kernel.endswith("fused>"):
        return n * (2 * N + 2 + 2 * N)
    if kernel.startswith("k_bf16_reduce"):
        return n * (2 * N + 2)
    if kernel == "k_broadcast":
        return n * (2 + 2 * N)
    raise ValueError(kernel)


def min_dram_bytes(codec, N, n):
    """The fewest DRAM bytes an emulated all-reduce call can move: every input
    read, every stage-1 wire and the gathered wire written once (they are the
    transmitted data), every output written; the wires' read-back may come from
    L2.  ncu DRAM bytes of the large workloads sit at this figure."""
    c = CODEC_C[codec]
    if codec == "bf16":
        return n * (2 * N + 2 + 2 * N)
    return N * n * (4 + c) + n * c


def min_dram_for(kernel, codec, N, n):
    """min_dram_bytes for the single-pass kernels (whose stage-1 read-back may
    hit L2); the algorithmic bytes for every other kernel."""
    c = CODEC_C[codec]
    if kernel.startswith("k_allreduce_single_f32"):
        return N * n * (4 + c) + n * c + 4 * N * n
    if kernel.startswith("k_allreduce_single") or kernel.startswith("k_allreduce_tile"):
        return min_dram_bytes(codec, N, n)
    return algorithmic_bytes(kernel, codec, N, n)


def traffic_for(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on these sources."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    sha = source_sha()
    with open(TRAFFIC_FILE) as f:
        for line in f:
            kv = dict(re.findall(r"(\w+)=(\S+)", line))
            if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("source_sha") == sha:
                return int(kv["bytes_per_launch"])
    return None


# ---- multi-rank aggregation (one process per GPU) -----------------------------------
def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank contributes, all receive the max."""
    if world <= 1:
        return float(ms)
    if torch.distributed.get_backend() == "gloo":
        device = torch.device("cpu")                  # gloo reduces host tensors
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world, bytes_per_rank_step, steps, ms_max):
    """Whole-job throughput: the bytes of every rank over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


# ---- clocks sampled during the timed region -------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- our arm -------------------------------------------------------------------------
def run_ours(args, device):
    """One GPU: the workload's N ranks emulated in its HBM."""
    from quantized_precision_all_b200 import lpar as L

    w = W.WORKLOADS[args.workload]
    N, n = w.N, w.n
    f32 = w.dtype == "f32"
    xs = W.make_inputs(w, device)

    def eff_codec(c):                        # the threshold compares message bytes
        return L.lpar_effective_codec(w.elem_bytes * n // 2, c, w.min_quant_bytes)

    if f32:
        ws_bytes = max(L.lpar_collective_workspace_bytes("allreduce_f32", N, n, eff_codec(c)) for c in w.codecs)
        allreduce = L.lpar_allreduce_f32
    else:
        ws_bytes = max(L.lpar_workspace_bytes(N, n, eff_codec(c)) for c in w.codecs)
        allreduce = L.lpar_allreduce
    stream = torch.cuda.current_stream(device)
    # Buffer sets at distinct addresses spanning at least 4x L2, rotated step by
    # step, so that every step reads its inputs from HBM (one set when the
    # workload alone exceeds that).
    sets = BufferSets(xs, n, ws_bytes, device, out_dtype=xs[0].dtype)
    R = sets.R

    def step(k=0, stage_events=None, st=None):
        i = k % R
        for j, codec in enumerate(w.codecs):
            allreduce(sets.inputs[i], n, codec, sets.outputs[i], sets.ws[i], sets.ws_bytes, w.min_quant_bytes,
                      args.schedule, st or stream, stage_events=None if stage_events is None else stage_events[j])

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize(device)

    # (1) the timed region: K steps, CUDA events on the launching stream; by
    # default the K steps are captured in one CUDA graph (the library allocates
    # and synchronises nothing, so its calls capture) and the graph is replayed
    # once untimed, then once timed: the host's per-call cost stays out of the
    # device timeline.  --eager issues the K steps from Python instead.
    graph = None
    if not args.eager:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for k in range(args.steps):
                step(k, st=side)
        stream.wait_stream(side)
        graph.replay()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clocks:
        start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for k in range(args.steps):
                step(k)
        end.record(stream)
        torch.cuda.synchronize(device)
    ms_total = start.elapsed_time(end)
    del graph

    # (2) per-kernel durations, live: stage events recorded between the kernels
    ksteps = max(1, min(args.steps, 200))
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in w.codecs] for _ in range(ksteps)]
    for per_step in evs:                     # torch creates the CUDA event on its first record()
        for per_codec in per_step:
            for ev in per_codec:
                ev.record(stream)
    torch.cuda.synchronize(device)
    for s in range(ksteps):
        step(s, evs[s])
    torch.cuda.synchronize(device)
    kern = {}
    for ci, codec in enumerate(w.codecs):
        eff = eff_codec(codec)
        names = kernel_names(eff, args.schedule, N, f32, n)
        if f32:
            bounds = [(0, 1)]
        elif eff == "bf16":
            bounds = [(1, 2), (2, 3)]
        elif args.schedule == "single_pass":
            bounds = [(0, 1)]
        else:
            bounds = [(0, 1), (1, 2), (2, 3)]
        for name, (a, b) in zip(names, bounds):
            tot = sum(evs[s][ci][a].elapsed_time(evs[s][ci][b]) for s in range(ksteps))
            d = kern.setdefault(name, {"codec": eff, "ms_total": 0.0, "launches": 0})
            d["ms_total"] += tot
            d["launches"] += ksteps
    for name, d in kern.items():
        d["ms_per_launch"] = d["ms_total"] / d["launches"]
        d["algorithmic_bytes"] = algorithmic_bytes(name, d["codec"], N, n)
        d["achieved_gbs"] = d["algorithmic_bytes"] / (d["ms_per_launch"] * 1e-3) / 1e9
        d["min_dram_bytes"] = min_dram_for(name, d["codec"], N, n)
    launches_per_step = sum(len(kernel_names(eff_codec(c), args.schedule, N, f32)) for c in w.codecs)

    # (3) accuracy of this step's outputs on sampled tiles (outside the timed region)
    accuracy = {}
    if not f32:
        T = n // TILE
        rng = torch.Generator().manual_seed(11)
        sample = torch.unique(torch.cat([torch.tensor([0, T - 1]), torch.randint(0, T, (62,), generator=rng)]))
        for codec in w.codecs:
            allreduce(sets.inputs[0], n, codec, sets.outputs[0], sets.ws[0], sets.ws_bytes, w.min_quant_bytes,
                      args.schedule, stream)
            torch.cuda.synchronize(device)
            accuracy[codec] = sample_check(xs, sets.outputs[0], sample.numpy())

    # (4) end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 5))
        h_in = [torch.empty(n, dtype=xs[0].dtype, pin_memory=True) for _ in range(N)]
        for h, x in zip(h_in, xs):
            h.copy_(x)
        h_out = [torch.empty(n, dtype=xs[0].dtype, pin_memory=True) for _ in range(N)]

        # the host all-reduce: chunks uploaded, reduced and downloaded on three
        # streams of the library, overlapped; one call per codec
        chunk = min(n, max(TILE, HOST_CHUNK_BYTES // (N * w.elem_bytes) // TILE * TILE))
        if f32:
            host_call, staging_bytes = L.lpar_allreduce_f32_host, L.lpar_host_staging_bytes_f32
        else:
            host_call, staging_bytes = L.lpar_allreduce_host, L.lpar_host_staging_bytes
        staging = torch.empty(max(staging_bytes(N, chunk, eff_codec(c)) for c in w.codecs), dtype=torch.uint8,
                              device=device)

        def e2e_step():
            for codec in w.codecs:
                host_call(h_in, n, codec, h_out, chunk, staging, staging.numel(), w.min_quant_bytes, args.schedule,
                          stream)
        h2d = N * w.elem_bytes * n * len(w.codecs)
        api = ("%s with pinned host buffers: chunks of %d elements per rank uploaded, reduced and downloaded on "
               "three streams, overlapped; one call per codec" % (host_call.__name__, chunk))

        e2e_step()
        torch.cuda.synchronize(device)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = s0.elapsed_time(s1)
        eb = w.elem_bytes
        e2e = {"value": aggregate_gbs(1, N * eb * n * len(w.codecs), e2e_steps, e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": N * eb * n * len(w.codecs),
               "steps": e2e_steps, "ms_per_step": e_ms / e2e_steps, "api": api}
        del h_in, h_out

    # (5) the oracle on the host cores (one GPU, one process)
    cpu = None if args.no_cpu_baseline else cpu_baseline(w, xs)

    return {"ms": ms_total, "kern": kern, "clocks": clocks.summary(), "launches_per_step": launches_per_step,
            "e2e": e2e, "cpu": cpu, "w": w, "accuracy": accuracy, "sets": R, "inputs": input_digests(w, xs)}


def input_digests(w, xs):
    """The seed and the SHA-256 of each rank's input bytes (host copy), so that a
    result row names the exact inputs it was measured on."""
    out = []
    for r, x in enumerate(xs):
        h = hashlib.sha256()
        flat = x.reshape(-1).view(torch.uint8)
        step = 256 << 20
        for i in range(0, flat.numel(), step):
            h.update(flat[i:i + step].cpu().numpy().tobytes())
        out.append({"rank": r, "seed": w.seed * 1009 + r, "sha256": h.hexdigest()})
    return out


def nvlink_bytes_sent(world, n, codec, chunks, rank=0):
    """Wire bytes one rank sends in one real all-reduce: its wire minus its own
    shard in the all-to-all, its padded send slot to every peer in the
    all-gather, chunk by chunk."""
    from quantized_precision_all_b200 import distributed as D
    tb = int(round(CODEC_C[codec] * TILE))
    total = 0
    for t0, t1 in D.chunk_tiles(n // TILE, chunks):
        shards = D.shard_tiles(world, t1 - t0)
        width = max(b - a for a, b in shards) * tb
        total += (t1 - t0) * tb - (shards[rank][1] - shards[rank][0]) * tb + (world - 1) * width
    return total


def peer_bytes_sent(world, n, codec, rank=0):
    """Wire bytes one rank stores into other ranks' memory in one peer-kernel
    all-reduce: its wire tiles of the other ranks' shards, and its reduced
    shard into every other rank's gathered wire (the flags aside)."""
    from quantized_precision_all_b200 import distributed as D
    tb = int(round(CODEC_C[codec] * TILE))
    T = n // TILE
    a, b = D.shard_tiles(world, T)[rank]
    return (T - (b - a)) * tb + (world - 1) * (b - a) * tb


def run_distributed(args, rank, world, device):
    """The real all-reduce across the `world` processes (one GPU each): rank r
    holds rank r's message of the workload (same size, same seeded recipe);
    each step runs every codec of the workload through DistributedAllreduce
    (--exchange nccl) or PeerAllreduce (--exchange peer)."""
    from quantized_precision_all_b200.distributed import DistributedAllreduce, PeerAllreduce
    w = W.WORKLOADS[args.workload]
    if w.dtype != "bf16":
        raise SystemExit("the cross-GPU all-reduce takes BF16 messages")
    n = w.n
    x = W.make_rank_input(w, rank, device)
    out = torch.empty_like(x)
    peer = args.exchange == "peer"
    ar = PeerAllreduce(device=device) if peer else DistributedAllreduce(chunks=args.chunks)
    stream = torch.cuda.current_stream(device)

    def step():
        for codec in w.codecs:
            ar.allreduce(x, codec, w.min_quant_bytes, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    torch.distributed.barrier()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(device)
    torch.distributed.barrier()
    ms_max = max_over_ranks(start.elapsed_time(end), world, device)

    def eff(c):
        return c if c == "bf16" or 2 * n >= w.min_quant_bytes else "bf16"

    if peer:
        ar.check()
        sent = sum(peer_bytes_sent(world, n, eff(c), rank) for c in w.codecs)
        launches = len(w.codecs)
    else:
        sent = sum(nvlink_bytes_sent(world, n, eff(c), args.chunks, rank) for c in w.codecs)
        launches = 0
        from quantized_precision_all_b200 import distributed as D
        for c in w.codecs:
            for t0, t1 in D.chunk_tiles(n // TILE, args.chunks):
                launches += 2 + sum(1 for a, b in D.shard_tiles(world, t1 - t0) if b > a)

    e2e = None
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 5))
        h_in = torch.empty(n, dtype=x.dtype, pin_memory=True)
        h_in.copy_(x)
        h_out = torch.empty(n, dtype=x.dtype, pin_memory=True)

        def e2e_step():
            for codec in w.codecs:
                x.copy_(h_in, non_blocking=True)
                ar.allreduce(x, codec, w.min_quant_bytes, out=out)
                h_out.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(device)
        torch.distributed.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        s1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = max_over_ranks(s0.elapsed_time(s1), world, device)
        per = 2 * n * len(w.codecs)
        e2e = {"value": aggregate_gbs(world, per, e2e_steps, e_ms), "unit": "GB/s", "h2d_bytes_per_step": per,
               "d2h_bytes_per_step": per, "steps": e2e_steps, "ms_per_step": e_ms / e2e_steps,
               "api": "%s.allreduce, each rank's message uploaded from pinned host memory and its result "
                      "downloaded, per codec" % type(ar).__name__}
        del h_in, h_out
    ar.release()
    return {"ms": ms_max, "clocks": clocks.summary(), "sent": sent, "launches_per_step": launches, "e2e": e2e,
            "w": w, "exchange": args.exchange}


def oracle_codecs(w):
    """The codecs the whole message runs with (the threshold compares the
    per-rank message bytes); oracle samples are then called with no threshold."""
    return [c if c == "bf16" or w.message_bytes >= w.min_quant_bytes else "bf16" for c in w.codecs]


def host_inputs(w, xs, tiles):
    """The first `tiles` tiles of each rank's input as the oracle takes them."""
    if w.dtype == "f32":
        return [x[:tiles * TILE].cpu().numpy() for x in xs]
    return [x[:tiles * TILE].view(torch.int16).cpu().numpy().view("uint16") for x in xs]


def cpu_baseline(w, xs_dev, tiles=CPU_BASELINE_TILES):
    """The oracle on the host: single-threaded on a sample of `tiles` tiles per
    rank, then over tile ranges on every host core (one worker process per
    core, PAR_TILES_PER_CORE tiles each).  The all-cores figure is the value."""
    from oracle import oracle as O, parallel as OP
    codecs = oracle_codecs(w)
    f32 = w.dtype == "f32"
    fn = O.allreduce_f32 if f32 else O.allreduce
    T = w.n // TILE
    tiles = min(tiles, T)
    xs = host_inputs(w, xs_dev, tiles)
    t0 = time.perf_counter()
    for codec in codecs:
        fn(xs, codec, 0)
    dt = time.perf_counter() - t0
    del xs
    single = {"value": w.N * w.elem_bytes * tiles * TILE * len(codecs) / dt / 1e9,
              "sample": "first %d tiles (%d MiB %s) of each of the %d ranks, codecs %s, %.1f s on one core"
                        % (tiles, tiles * TILE * w.elem_bytes >> 20, w.dtype.upper(), w.N, "+".join(codecs), dt)}
    cores = OP.host_cores()
    ptiles = min(T, cores * PAR_TILES_PER_CORE)
    dp, used = OP.run(host_inputs(w, xs_dev, ptiles), codecs, f32=f32, workers=cores)
    return {"value": w.N * w.elem_bytes * ptiles * TILE * len(codecs) / dp / 1e9, "unit": "GB/s", "cores": used,
            "kind": "oracle",
            "sample": "first %d tiles (%d MiB %s) of each of the %d ranks, codecs %s, split over %d worker "
                      "processes (one per host core), %.2f s from the common start to the last end"
                      % (ptiles, ptiles * TILE * w.elem_bytes >> 20, w.dtype.upper(), w.N, "+".join(codecs), used, dp),
            "single_core": single}


# ---- reference arm: the oracle as it stands, on the host --------------------------
def run_reference(args):
    """The oracle on every host core (tile ranges, one worker process per
    core), REF_TILES_PER_STEP tiles per rank per worker per step."""
    from oracle import parallel as OP
    w = W.WORKLOADS[args.workload]
    f32 = w.dtype == "f32"
    codecs = oracle_codecs(w)
    cores = OP.host_cores()
    tiles = min(cores * REF_TILES_PER_STEP, w.n // TILE)
    xs = host_inputs(w, W.make_inputs(w, "cpu", n=tiles * TILE), tiles)
    dt, used = OP.run(xs, codecs, f32=f32, workers=cores, warmup=args.warmup, repeat=max(args.steps, 1))
    value = w.N * w.elem_bytes * tiles * TILE * len(codecs) * max(args.steps, 1) / dt / 1e9
    sample = "%d tiles (%d KiB %s) per rank per step of workload %s, codecs %s, over %d worker processes" % (
        tiles, tiles * TILE * w.elem_bytes >> 10, w.dtype.upper(), w.name, "+".join(codecs), used)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": used, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def sample_check(xs, outs, tiles):
    """The error of sampled output tiles against the exact (binary64) sum of the
    inputs, and a hash of the sampled input bytes.  Bit-exact parity with the
    oracle on the same points is the business of tests/test_gpu_parity.py
    (test_workload_large_sampled_tiles, test_sweep_sampled_tiles)."""
    idx = torch.from_numpy((tiles[:, None] * TILE + torch.arange(TILE).numpy()[None, :]).reshape(-1)).to(xs[0].device)
    ins = [x[idx].float().cpu().numpy().astype("float64") for x in xs]     # BF16 -> binary64 is exact
    got = outs[0][idx].float().cpu().numpy().astype("float64")
    err = got - sum(ins)
    h = hashlib.blake2b(digest_size=8)
    for x in xs:
        h.update(x[idx].view(torch.int16).cpu().numpy().tobytes())
    return {"sampled_tiles": int(len(tiles)), "max_abs_err_vs_exact": float(abs(err).max()),
            "rms_err_vs_exact": float((err ** 2).mean() ** 0.5), "input_sample_blake2b": h.hexdigest()}


def oracle_gbs(op, N, codec, tiles=64):
    """The oracle's rate on a small seeded sample (its cost per tile does not
    depend on the message size): GB/s of N x per-rank message bytes, one core."""
    from oracle import oracle as O
    w = W.Workload("oracle_sample", N=N, n=tiles * TILE, dist="student_t", nu=3, seed=9, codecs=(codec,))
    xs = [x.view(torch.int16).numpy().view("uint16") for x in W.make_inputs(w, "cpu")]
    fn = {"allreduce": O.allreduce, "reduce_scatter": O.reduce_scatter, "one_shot": O.allreduce_oneshot,
          "all_gather": O.all_gather, "all_to_all": O.all_to_all, "peer_allreduce": O.allreduce}[op]
    t0 = time.perf_counter()
    fn(xs, codec)
    dt = time.perf_counter() - t0
    return {"value": N * 2 * tiles * TILE / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d tiles per rank, N=%d, %s, %s" % (tiles, N, codec, op)}


class BufferSets:
    """R copies of one call's buffers (inputs, outputs, workspace) at distinct
    addresses, R chosen so that the sets span at least ROTATE_BYTES (4x L2):
    calls that rotate over them find their inputs outside L2 even when timed
    back to back."""

    def __init__(self, xs, out_elems, ws_bytes, device, rotate=ROTATE_BYTES, out_dtype=torch.bfloat16):
        N, n = len(xs), xs[0].numel()
        wsb = -(-max(ws_bytes, 16) // 256) * 256
        out_size = torch.empty(0, dtype=out_dtype).element_size()
        set_bytes = N * n * xs[0].element_size() + N * out_elems * out_size + wsb
        self.R = max(1, -(-rotate // set_bytes))
        if self.R == 1:
            self.inputs = [list(xs)]
        else:
            pool = torch.empty((self.R, N, n), dtype=xs[0].dtype, device=device)
            pool[:] = torch.stack(list(xs))
            self.inputs = [list(pool[i].unbind(0)) for i in range(self.R)]
        outs = torch.empty((self.R, N, out_elems), dtype=out_dtype, device=device)
        self.outputs = [list(outs[i].unbind(0)) for i in range(self.R)]
        ws = torch.empty((self.R, wsb), dtype=torch.uint8, device=device)
        self.ws = [ws[i] for i in range(self.R)]
        self.ws_bytes = wsb


def time_call(call, R, flush, device, single_iters=20, batches=3):
    """Per-call time of call(i, stream) for buffer set i, in microseconds, two ways:
    single: one call between two CUDA events after a 256 MiB write (cold L2),
    median of single_iters; graph: K calls rotating over the R sets captured in
    one CUDA graph and replayed (launches pipelined, no host enqueue cost in the
    timed region), replay time / K, median of `batches` replays.  CUDA events on
    this pool tick in steps of about 2.05 us, so the single-call figure carries
    that resolution and the graph figure resolves it away."""
    stream = torch.cuda.current_stream(device)
    for i in range(min(R, 3)):
        call(i, stream)
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(single_iters)]
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        call(0, stream)
        e1.record(stream)
    torch.cuda.synchronize(device)
    single = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs) * 1e3
    K = min(max(2 * R, 20), 4000)
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for k in range(K):
            call(k % R, side)
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize(device)
    per = []
    for _ in range(batches):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        per.append(e0.elapsed_time(e1) * 1e3 / K)
    del g
    return {"us_single": single, "us": statistics.median(per), "us_min": min(per), "calls_per_graph": K}


def _fractions(alg, dram, N, mb, us, peak):
    t = us * 1e-6
    return {"GBps": N * mb / t / 1e9, "hbm_fraction": alg / t / 1e9 / peak, "dram_fraction": dram / t / 1e9 / peak}


def run_sweep(args, device):
    """One JSON line per sweep point (N, message size, codec): GB/s and the
    fraction of measured HBM peak the whole call reaches, per call back to back
    (CUDA graph over rotating buffer sets) and as a single cold call, with the
    SM clock record of the (N, size) group."""
    from quantized_precision_all_b200 import lpar as L
    peak, peak_src = measured_peaks()
    ranks = [args.sweep_n] if args.sweep_n else list(W.SWEEP_RANKS)
    sizes = [args.sweep_mib << 20] if args.sweep_mib else list(W.SWEEP_SIZES_BYTES)
    codecs = [args.sweep_codec] if args.sweep_codec else list(W.SWEEP_CODECS)
    cpu = {(N, c): oracle_gbs("allreduce", N, c) for N in ranks for c in codecs}
    done = set()
    if args.resume and os.path.exists(args.resume):   # restart: skip the points already written
        with open(args.resume) as f:
            for line in f:
                if line.startswith("{"):
                    d = json.loads(line)
                    done.add((d["N"], d["message_bytes"], d["codec"]))
    sink = open(args.resume, "a") if args.resume else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)   # > L2, rewritten before single calls
    for N in ranks:
        for mb in sizes:
            todo = [c for c in codecs if (N, mb, c) not in done]
            if not todo:
                continue
            w = W.sweep_workload(N, mb, "bf16")
            xs = W.make_inputs(w, device)
            wsb = max(L.lpar_workspace_bytes(N, w.n, c) for c in todo)
            sets = BufferSets(xs, w.n, wsb, device)
            T = w.n // TILE
            rng = torch.Generator().manual_seed(5000 + N)
            sample = torch.unique(torch.cat([torch.tensor([0, T - 1]), torch.randint(0, T, (2,), generator=rng)]))
            rows = []
            with ClockSampler(device) as clocks:
                for codec in todo:
                    def call(i, st, codec=codec):
                        L.lpar_allreduce(sets.inputs[i], w.n, codec, sets.outputs[i], sets.ws[i], sets.ws_bytes,
                                         schedule=args.schedule, stream=st)
                    tm = time_call(call, sets.R, flush, device)
                    names = kernel_names(codec, args.schedule, N, n=w.n)
                    alg = sum(algorithmic_bytes(k, codec, N, w.n) for k in names)
                    dram = min_dram_bytes(codec, N, w.n)
                    graph = _fractions(alg, dram, N, mb, tm["us"], peak)
                    single = _fractions(alg, dram, N, mb, tm["us_single"], peak)
                    call(0, torch.cuda.current_stream(device))
                    torch.cuda.synchronize(device)
                    rows.append({"sweep": True, "N": N, "message_bytes": mb, "codec": codec,
                                 "schedule": args.schedule, "kernel": names[0],
                                 "us": tm["us"], "us_single": tm["us_single"], "ms": tm["us"] * 1e-3,
                                 **graph, **{k + "_single": v for k, v in single.items()},
                                 "algorithmic_bytes": alg, "min_dram_bytes": dram,
                                 "rotated_sets": sets.R, "calls_per_graph": tm["calls_per_graph"],
                                 "timing": "us: K calls over the rotated buffer sets in one CUDA graph, replay "
                                           "time / K (inputs outside L2); us_single: one call after a 256 MiB "
                                           "write, median of 20",
                                 "peak": peak, "cpu_baseline": cpu[(N, codec)], "seed": w.seed,
                                 **sample_check(xs, sets.outputs[0], sample.numpy())})
            clk = clocks.summary()
            for row in rows:
                row["clocks"] = clk
                line = json.dumps(row)
                print(line, flush=True)
                if sink:
                    sink.write(line + "\n")
                    sink.flush()
            del xs, sets
            torch.cuda.empty_cache()


def run_floor(args, device):
    """Small messages against the per-call floor: the same call with a one-tile
    BF16 message on one rank (one tiny kernel through lpar_allreduce), then the
    all-reduce of 128 KiB - 2 MiB per rank; each timed single (cold) and back to
    back (CUDA graph), and back to back from Python (eager enqueue)."""
    from quantized_precision_all_b200 import lpar as L
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def eager(call, R, K=200):
        for i in range(3):
            call(i % R, stream)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k in range(K):
            call(k % R, stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) * 1e3 / K

    points = [(1, 2048 * 2, "bf16", "floor: one tile on one rank, BF16")]
    for N in (2, 4, 8):
        for mb in (128 << 10, 256 << 10, 512 << 10, 1 << 20, 2 << 20):
            for codec in W.SWEEP_CODECS:
                points.append((N, mb, codec, ""))
    with ClockSampler(device) as clocks:
        rows = []
        for N, mb, codec, note in points:
            w = W.sweep_workload(N, mb, "bf16")
            xs = W.make_inputs(w, device)
            wsb = L.lpar_workspace_bytes(N, w.n, codec)
            sets = BufferSets(xs, w.n, wsb, device)

            def call(i, st):
                L.lpar_allreduce(sets.inputs[i], w.n, codec, sets.outputs[i], sets.ws[i], sets.ws_bytes,
                                 schedule=args.schedule, stream=st)
            tm = time_call(call, sets.R, flush, device)
            rows.append({"floor": True, "N": N, "message_bytes": mb, "codec": codec, "note": note,
                         "us_graph": tm["us"], "us_single": tm["us_single"], "us_eager": eager(call, sets.R),
                         "GBps_graph": N * mb / (tm["us"] * 1e-6) / 1e9})
            del xs, sets
    clk = clocks.summary()
    for row in rows:
        row["clocks"] = clk
        print(json.dumps(row), flush=True)


COLL_OPS = ("reduce_scatter", "one_shot", "all_gather", "all_to_all", "peer_allreduce")
COLL_SIZES_BYTES = (16 << 20, 256 << 20)             # per-rank message


def collective_bytes(op, codec, N, size):
    """Algorithmic HBM bytes of one collective call.  size = elements of the size
    argument (reduce-scatter / one-shot: n per rank; all-gather: m per rank;
    all-to-all: m per segment, N * m per rank; the peer-memory all-reduce: n per
    rank).  Quantising codecs: the N messages are read and their wires written;
    reductions read the N wires back and write one (reduce-scatter) or N
    (one-shot) BF16 results; all-gather and all-to-all decode from the encoder's
    registers and write the outputs.  The peer-memory all-reduce with every rank
    in one GPU moves each stage through memory: the N messages read, the N
    wires written into the mailboxes and read back, the reduced wire written
    into all N gathered wires and read back, the N outputs written."""
    c = CODEC_C[codec]
    if op == "peer_allreduce":
        return N * size * (4 + 4 * c)
    msg = N * size if op == "all_to_all" else size        # per-rank message, elements
    out = {"reduce_scatter": 2 * size, "one_shot": N * 2 * size,
           "all_gather": N * N * 2 * size, "all_to_all": N * N * 2 * size}[op]
    if codec == "bf16":
        return N * 2 * msg + out
    stage1 = N * msg * (2 + c)
    back = N * msg * c if op in ("reduce_scatter", "one_shot") else 0
    return stage1 + back + out


def run_collectives(args, device):
    """One JSON line per (op, N, message size, codec) of the standalone
    collectives and the one-shot all-reduce: GB/s (N x per-rank message bytes
    / time) and the fraction of measured HBM peak (algorithmic bytes / time),
    back to back (CUDA graph over rotating buffer sets) and as a single cold
    call, with the SM clock record of the (op, N, size) group."""
    from quantized_precision_all_b200 import lpar as L
    peak, _ = measured_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    ops = [args.coll_op] if args.coll_op else COLL_OPS
    ranks = [args.coll_n] if args.coll_n else (2, 4, 8)
    sizes = [args.coll_mib << 20] if args.coll_mib else COLL_SIZES_BYTES
    codecs = [args.coll_codec] if args.coll_codec else W.SWEEP_CODECS
    cpu = {(op, N, c): oracle_gbs(op, N, c) for op in ops for N in ranks for c in codecs}
    for op in ops:
        for N in ranks:
            for mb in sizes:
                msg = mb // 2
                size = msg // N if op == "all_to_all" else msg
                w = W.Workload("collective", N=N, n=msg, dist="student_t", nu=3, seed=9, codecs=("bf16",))
                xs = W.make_inputs(w, device)
                if op == "all_gather":
                    xs = [x[:size] for x in xs]
                out_elems = N * size if op in ("all_gather", "all_to_all") else msg
                if op == "peer_allreduce":                 # mailboxes + gathered wires of the N ranks
                    wsb = max(N * (L.lpar_peer_mailbox_bytes(N, msg, c) + L.lpar_peer_gather_bytes(msg, c))
                              for c in codecs)
                else:
                    wsb = max(L.lpar_workspace_bytes(N, msg, c) for c in codecs)
                sets = BufferSets(xs, out_elems, wsb, device)
                rows = []
                with ClockSampler(device) as clocks:
                    for codec in codecs:
                        peer = ([L.PeerBuffers(N, msg, codec, device) for _ in range(sets.R)]
                                if op == "peer_allreduce" else None)

                        def call(i, st, codec=codec, peer=peer):
                            if op == "peer_allreduce":
                                peer[i].allreduce(sets.inputs[i], sets.outputs[i], stream=st)
                            elif op == "one_shot":
                                L.lpar_allreduce(sets.inputs[i], msg, codec, sets.outputs[i], sets.ws[i],
                                                 sets.ws_bytes, schedule="one_shot", stream=st)
                            else:
                                getattr(L, "lpar_" + op)(sets.inputs[i], size, codec, sets.outputs[i], sets.ws[i],
                                                         sets.ws_bytes, stream=st)
                        tm = time_call(call, sets.R, flush, device, single_iters=10)
                        alg = collective_bytes(op, codec, N, size)
                        rows.append({"collective": op, "N": N, "message_bytes": mb, "codec": codec,
                                     "us": tm["us"], "us_single": tm["us_single"], "ms": tm["us"] * 1e-3,
                                     "GBps": N * mb / (tm["us"] * 1e-6) / 1e9,
                                     "GBps_single": N * mb / (tm["us_single"] * 1e-6) / 1e9,
                                     "hbm_fraction": alg / (tm["us"] * 1e-6) / 1e9 / peak,
                                     "hbm_fraction_single": alg / (tm["us_single"] * 1e-6) / 1e9 / peak,
                                     "algorithmic_bytes": alg, "peak": peak, "cpu_baseline": cpu[(op, N, codec)],
                                     "rotated_sets": sets.R, "calls_per_graph": tm["calls_per_graph"]})
                        if peer:
                            for b in peer:
                                b.check()
                            del peer
                clk = clocks.summary()
                for row in rows:
                    row["clocks"] = clk
                    print(json.dumps(row), flush=True)
                del xs, sets
                torch.cuda.empty_cache()


def emulation_config(w, args, sets, inputs=None):
    cfg = workload_config(w, args)
    if inputs:
        cfg["inputs"] = inputs
    if sets > 1:
        cfg["l2"] = ("inputs %d MiB < 4x L2: the steps rotate over %d buffer sets at distinct addresses spanning "
                     ">= %d MiB, so every step reads its inputs from HBM" % (w.N * w.message_bytes >> 20, sets,
                                                                              ROTATE_BYTES >> 20))
    cfg["timing"] = ("the K timed steps issued from Python" if args.eager else
                     "the K timed steps captured in one CUDA graph, replayed once untimed, then once timed")
    return cfg


def workload_config(w, args, world=1):
    cfg = {"workload": w.name, "simulated_ranks": w.N, "elements_per_rank": w.n, "message_dtype": w.dtype,
           "message_bytes_per_rank": w.message_bytes, "codecs": list(w.codecs), "schedule": args.schedule,
           "distribution": w.note, "min_quant_bytes": w.min_quant_bytes,
           "l2": "inputs %d MiB > 126 MB L2: no flush between steps" % (w.N * w.message_bytes >> 20)
           if w.N * w.message_bytes > 126e6 else "inputs fit in L2",
           "parallelism": "the %d ranks simulated in one GPU's HBM (emulated reduce-scatter / all-gather)" % w.N}
    if world > 1:
        peer = getattr(args, "exchange", "nccl") == "peer"
        cfg.update({"simulated_ranks": None, "ranks": world, "exchange": "peer" if peer else "nccl",
                    "l2": "message %d MiB per rank > 126 MB L2: no flush between steps" % (w.message_bytes >> 20),
                    "parallelism": ("real all-reduce across %d GPUs, one rank per GPU: one peer-memory kernel per "
                                    "rank storing wire tiles into the other ranks' memory over CUDA IPC" % world)
                    if peer else
                    ("real all-reduce across %d GPUs, one rank per GPU: the library's stage kernels with %s "
                     "all-to-all and all-gather of the wire bytes, %d chunk(s) pipelined"
                     % (world, args.backend.upper(), args.chunks))})
    return cfg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_int3_int4", choices=sorted(W.WORKLOADS))
    ap.add_argument("--schedule", default="auto", choices=["auto", "fused", "three_stage", "single_pass"])
    ap.add_argument("--chunks", type=int, default=4,
                    help="with --gpus > 1: tile ranges pipelined through the cross-GPU all-reduce")
    ap.add_argument("--exchange", choices=["nccl", "peer"], default="nccl",
                    help="with --gpus > 1: NCCL exchanges between the stage kernels (DistributedAllreduce) or "
                         "one peer-memory kernel per rank over CUDA IPC (PeerAllreduce; GPUs must be distinct)")
    ap.add_argument("--backend", choices=["nccl", "gloo"], default="nccl",
                    help="with --gpus > 1: the process group's backend (gloo moves the wire bytes through host "
                         "copies; for testing the multi-rank path on fewer GPUs than ranks)")
    ap.add_argument("--eager", action="store_true",
                    help="issue the timed steps from Python instead of replaying them from one CUDA graph")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="one JSON line per sweep point instead of the bench line")
    ap.add_argument("--sweep-n", type=int, default=None, help="with --sweep: only this N")
    ap.add_argument("--sweep-mib", type=int, default=None, help="with --sweep: only this per-rank MiB size")
    ap.add_argument("--sweep-codec", default=None, help="with --sweep: only this codec")
    ap.add_argument("--resume", default=None,
                    help="with --sweep: append rows to this JSONL file and skip the points it already holds")
    ap.add_argument("--collectives", action="store_true",
                    help="one JSON line per standalone collective point instead of the bench line")
    ap.add_argument("--coll-op", choices=list(COLL_OPS), default=None,
                    help="with --collectives: only this collective")
    ap.add_argument("--coll-n", type=int, default=None, help="with --collectives: only this N")
    ap.add_argument("--coll-mib", type=int, default=None, help="with --collectives: only this per-rank MiB size")
    ap.add_argument("--coll-codec", default=None, help="with --collectives: only this codec")
    ap.add_argument("--floor", action="store_true",
                    help="small messages against the per-call floor, one JSON line per point")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.chunks = max(1, args.chunks)
    if args.schedule == "auto":                # what the library picks for LPAR_SCHEDULE_AUTO
        args.schedule = "single_pass"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    device = torch.device("cuda", local_rank % max(1, torch.cuda.device_count()))
    torch.cuda.set_device(device)
    if args.sweep:
        run_sweep(args, device)
        return
    if args.collectives:
        run_collectives(args, device)
        return
    if args.floor:
        run_floor(args, device)
        return
    if world > 1:
        import datetime
        if args.backend == "nccl":
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=device)
        else:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        try:
            res = run_distributed(args, rank, world, device)
            if rank == 0:
                print(json.dumps(distributed_line(args, world, res)), flush=True)
            torch.distributed.barrier()
        finally:
            torch.distributed.destroy_process_group()
        return
    res = run_ours(args, device)
    print(json.dumps(emulation_line(args, res)), flush=True)


def distributed_line(args, world, res):
    w = res["w"]
    ms_per_step = res["ms"] / args.steps
    achieved = res["sent"] / (ms_per_step * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": aggregate_gbs(world, w.message_bytes * len(w.codecs), args.steps, res["ms"]),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, args, world),
        "roofline": {"bound": "nvlink", "kernel": ("whole step (one peer-memory kernel per codec)"
                                                   if res["exchange"] == "peer" else
                                                   "whole step (stage kernels and NCCL exchanges)"),
                     "achieved": achieved, "peak": NVLINK_GBS, "unit": "GB/s", "frac": achieved / NVLINK_GBS,
                     "traffic": None, "algorithmic_bytes_per_step": res["sent"],
                     "peak_source": "measured peer copy per direction per GPU on this pool (not MEASURED_PEAKS.json)"},
        "gpu_launches": res["launches_per_step"] * args.steps, "clocks": res["clocks"], "e2e": res["e2e"],
        "cpu_baseline": None, "source_sha": source_sha(),
    }


def emulation_line(args, res):
    w = res["w"]
    peak, peak_src = measured_peaks()
    step_bytes = w.N * w.message_bytes * len(w.codecs)
    ms_per_step = res["ms"] / args.steps
    value = aggregate_gbs(1, step_bytes, args.steps, res["ms"])
    kern = res["kern"]
    dom = max(kern, key=lambda k: kern[k]["ms_total"])
    total_ms = sum(d["ms_total"] for d in kern.values())
    alg_step = sum(d["algorithmic_bytes"] * d["launches"] for d in kern.values()) / (
        max(d["launches"] for d in kern.values()))
    d = kern[dom]
    traffic = traffic_for(dom, w.name)
    sec = d["ms_per_launch"] * 1e-3
    return {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": emulation_config(w, args, res["sets"], res.get("inputs")),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": d["achieved_gbs"], "peak": peak,
                     "unit": "GB/s", "frac": d["achieved_gbs"] / peak, "traffic": traffic,
                     "frac_dram": None if traffic is None else traffic / sec / 1e9 / peak,
                     "frac_min_dram": d["min_dram_bytes"] / sec / 1e9 / peak,
                     "algorithmic_bytes_per_launch": d["algorithmic_bytes"],
                     "min_dram_bytes_per_launch": d["min_dram_bytes"],
                     "ms_per_launch": d["ms_per_launch"], "share_of_step": d["ms_total"] / total_ms,
                     "peak_source": peak_src,
                     "basis": "frac: the schedule's algorithmic bytes (stage-1 wires written and read back); "
                              "frac_dram: ncu DRAM bytes per launch (null unless captured on these sources); "
                              "frac_min_dram: the fewest DRAM bytes a call can move (wire read-back from L2)"},
        "step_hbm_fraction": alg_step / (ms_per_step * 1e-3) / 1e9 / peak,
        "kernels": {k: {"ms_per_launch": v["ms_per_launch"], "achieved_gbs": v["achieved_gbs"],
                        "frac": v["achieved_gbs"] / peak, "share": v["ms_total"] / total_ms,
                        "algorithmic_bytes": v["algorithmic_bytes"]} for k, v in kern.items()},
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": res["clocks"],
        "e2e": res["e2e"],
        "cpu_baseline": res["cpu"],
        "accuracy": res["accuracy"],
        "source_sha": source_sha(),
    }


if __name__ == "__main__":
    main()
