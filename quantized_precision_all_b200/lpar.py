"""Python binding of the C ABI in ``include/lpar.h`` (argument marshalling only).

Every function has the C name and forwards to ``liblpar.so``; all arithmetic
runs in the library's CUDA kernels.  Device buffers may be given as CUDA
``torch.Tensor`` objects (contiguous) or as raw integer device addresses;
pointer arrays are Python sequences.  ``stream`` defaults to PyTorch's current
stream on the current device.

A call that returns a status other than LPAR_OK raises :class:`LparError`.
If the library has not been built, importing it raises ``OSError`` -- there is
no fallback implementation.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblpar.so")

LPAR_CODEC_BF16, LPAR_CODEC_FP8_E4M3, LPAR_CODEC_INT4, LPAR_CODEC_INT3, LPAR_CODEC_MXFP4 = 0, 1, 2, 3, 4
CODECS = {"bf16": LPAR_CODEC_BF16, "fp8": LPAR_CODEC_FP8_E4M3, "int4": LPAR_CODEC_INT4, "int3": LPAR_CODEC_INT3,
          "mxfp4": LPAR_CODEC_MXFP4}
CODEC_NAMES = {v: k for k, v in CODECS.items()}
LPAR_SCHEDULE_AUTO, LPAR_SCHEDULE_FUSED, LPAR_SCHEDULE_THREE_STAGE, LPAR_SCHEDULE_SINGLE_PASS = 0, 1, 2, 3
LPAR_SCHEDULE_ONE_SHOT = 4
SCHEDULES = {"auto": LPAR_SCHEDULE_AUTO, "fused": LPAR_SCHEDULE_FUSED, "three_stage": LPAR_SCHEDULE_THREE_STAGE,
             "single_pass": LPAR_SCHEDULE_SINGLE_PASS, "one_shot": LPAR_SCHEDULE_ONE_SHOT}
OPS = {"allreduce": 0, "reduce_scatter": 1, "all_gather": 2, "all_to_all": 3, "allreduce_f32": 4}
STATUS = {0: "LPAR_OK", 1: "LPAR_ERR_INVALID_ARG", 2: "LPAR_ERR_MISALIGNED",
          3: "LPAR_ERR_WORKSPACE_TOO_SMALL", 4: "LPAR_ERR_UNSUPPORTED", 5: "LPAR_ERR_CUDA"}
TILE_ELEMS = 2048
MAX_RANKS = 8

EXPORTS = ("lpar_tile_bytes", "lpar_wire_bytes", "lpar_workspace_bytes", "lpar_quantize", "lpar_reduce",
           "lpar_decode", "lpar_allreduce", "lpar_allreduce_static", "lpar_effective_codec", "lpar_status_string",
           "lpar_collective_workspace_bytes", "lpar_reduce_scatter", "lpar_all_gather", "lpar_all_to_all",
           "lpar_allreduce_f32", "lpar_host_staging_bytes", "lpar_allreduce_host", "lpar_host_staging_bytes_f32",
           "lpar_allreduce_f32_host", "lpar_peer_mailbox_bytes", "lpar_peer_gather_bytes", "lpar_peer_flag_bytes",
           "lpar_allreduce_peer", "lpar_peer_alloc", "lpar_peer_free", "lpar_peer_export", "lpar_peer_import",
           "lpar_peer_close")
LPAR_STATIC_WORKSPACE_BYTES = 16 << 20
LPAR_PEER_STATUS_WORDS = 8
LPAR_PEER_HANDLE_BYTES = 64


class LparError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib.lpar_status_string(status).decode()})")


class lpar_options_t(ctypes.Structure):
    _fields_ = [("min_quant_bytes", ctypes.c_size_t), ("schedule", ctypes.c_int),
                ("stage_events", ctypes.c_void_p * 4)]


def _load():
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    vpp = ctypes.POINTER(ctypes.c_void_p)
    sigs = {
        "lpar_tile_bytes": (sz, [i32]),
        "lpar_wire_bytes": (sz, [i32, sz]),
        "lpar_workspace_bytes": (sz, [i32, sz, i32]),
        "lpar_quantize": (i32, [vp, sz, i32, vp, vp]),
        "lpar_reduce": (i32, [vpp, i32, sz, sz, i32, vp, vp]),
        "lpar_decode": (i32, [vp, sz, i32, vp, vp]),
        "lpar_allreduce": (i32, [vpp, i32, sz, i32, vpp, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_allreduce_static": (i32, [vpp, i32, sz, i32, vpp, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_effective_codec": (i32, [sz, i32, ctypes.POINTER(lpar_options_t)]),
        "lpar_status_string": (ctypes.c_char_p, [i32]),
        "lpar_collective_workspace_bytes": (sz, [i32, i32, sz, i32]),
        "lpar_reduce_scatter": (i32, [vpp, i32, sz, i32, vpp, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_all_gather": (i32, [vpp, i32, sz, i32, vpp, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_all_to_all": (i32, [vpp, i32, sz, i32, vpp, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_allreduce_f32": (i32, [vpp, i32, sz, i32, vpp, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_host_staging_bytes": (sz, [i32, sz, i32]),
        "lpar_allreduce_host": (i32, [vpp, i32, sz, i32, vpp, sz, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_host_staging_bytes_f32": (sz, [i32, sz, i32]),
        "lpar_allreduce_f32_host": (i32, [vpp, i32, sz, i32, vpp, sz, vp, sz, ctypes.POINTER(lpar_options_t), vp]),
        "lpar_peer_mailbox_bytes": (sz, [i32, sz, i32]),
        "lpar_peer_gather_bytes": (sz, [sz, i32]),
        "lpar_peer_flag_bytes": (sz, [i32, sz]),
        "lpar_allreduce_peer": (i32, [vpp, vpp, vpp, vpp, vpp, i32, i32, i32, sz, i32, ctypes.c_uint64, vp, vp]),
        "lpar_peer_alloc": (i32, [sz, vpp]),
        "lpar_peer_free": (i32, [vp]),
        "lpar_peer_export": (i32, [vp, ctypes.c_char_p]),
        "lpar_peer_import": (i32, [ctypes.c_char_p, vpp]),
        "lpar_peer_close": (i32, [vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def library():
    """The loaded ctypes library (for symbol checks)."""
    return _lib


# ---- marshalling helpers ------------------------------------------------------
def _codec(c):
    return CODECS[c] if isinstance(c, str) else int(c)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("lpar: tensors must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError("lpar: tensors must be contiguous")
    return x.data_ptr()


_PTR_ARRAY_TYPES = [ctypes.c_void_p * k for k in range(MAX_RANKS + 1)]


def _ptr_array(xs, conv=None):
    """A ctypes array of the buffers' addresses; ctypes passes it where the C
    function takes `void *const *`."""
    if xs is None:
        return None
    conv = conv or _ptr
    k = len(xs)
    typ = _PTR_ARRAY_TYPES[k] if k <= MAX_RANKS else ctypes.c_void_p * k
    return typ(*[conv(x) for x in xs])


def _host_ptr(x):
    if x is None or isinstance(x, int):
        return x
    if x.is_cuda:
        raise ValueError("lpar: host buffers must live in host memory")
    if not x.is_contiguous():
        raise ValueError("lpar: tensors must be contiguous")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _options(min_quant_bytes=0, schedule="auto", stage_events=None):
    sched = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    opts = lpar_options_t(min_quant_bytes, sched)
    for i, ev in enumerate(stage_events or ()):
        if ev is not None:
            opts.stage_events[i] = ev if isinstance(ev, int) else ev.cuda_event
    return opts


def _check(status, where):
    if status != 0:
        raise LparError(status, where)


# ---- the C ABI ------------------------------------------------------------------
def lpar_tile_bytes(codec):
    return _lib.lpar_tile_bytes(_codec(codec))


def lpar_wire_bytes(codec, n):
    return _lib.lpar_wire_bytes(_codec(codec), n)


def lpar_workspace_bytes(N, n, codec):
    return _lib.lpar_workspace_bytes(N, n, _codec(codec))


def lpar_effective_codec(n, codec, min_quant_bytes=0):
    opts = _options(min_quant_bytes)
    return CODEC_NAMES[_lib.lpar_effective_codec(n, _codec(codec), ctypes.byref(opts))]


def lpar_quantize(in_bf16, n, codec, wire, stream=None):
    _check(_lib.lpar_quantize(_ptr(in_bf16), n, _codec(codec), _ptr(wire), _stream(stream)), "lpar_quantize")


def lpar_reduce(wires, tile_begin, tile_count, codec, wire_out, stream=None):
    arr = _ptr_array(wires)
    _check(_lib.lpar_reduce(arr, len(wires) if wires is not None else 0, tile_begin,
                            tile_count, _codec(codec), _ptr(wire_out), _stream(stream)), "lpar_reduce")


def lpar_decode(wire, n, codec, out_bf16, stream=None):
    _check(_lib.lpar_decode(_ptr(wire), n, _codec(codec), _ptr(out_bf16), _stream(stream)), "lpar_decode")


def lpar_allreduce(inputs, n, codec, out, workspace, workspace_bytes, min_quant_bytes=0, schedule="auto",
                   stream=None, N=None, stage_events=None):
    ins = _ptr_array(inputs)
    outs = _ptr_array(out)
    N = len(inputs) if N is None else N
    opts = _options(min_quant_bytes, schedule, stage_events)
    _check(_lib.lpar_allreduce(ins, N, n, _codec(codec), outs,
                               _ptr(workspace), workspace_bytes, ctypes.byref(opts), _stream(stream)),
           "lpar_allreduce")


def lpar_allreduce_static(inputs, n, codec, out, min_quant_bytes=0, schedule="auto", stream=None, N=None):
    """lpar_allreduce with the library's own 16 MiB workspace (no allocation)."""
    ins = _ptr_array(inputs)
    outs = _ptr_array(out)
    N = len(inputs) if N is None else N
    opts = _options(min_quant_bytes, schedule)
    _check(_lib.lpar_allreduce_static(ins, N, n, _codec(codec), outs,
                                      ctypes.byref(opts), _stream(stream)), "lpar_allreduce_static")


def lpar_allreduce_f32(inputs, n, codec, out, workspace, workspace_bytes, min_quant_bytes=0, schedule="auto",
                       stream=None, N=None, stage_events=None):
    """All-reduce of N binary32 messages (binary32 results)."""
    ins = _ptr_array(inputs)
    outs = _ptr_array(out)
    N = len(inputs) if N is None else N
    opts = _options(min_quant_bytes, schedule, stage_events)
    _check(_lib.lpar_allreduce_f32(ins, N, n, _codec(codec), outs,
                                   _ptr(workspace), workspace_bytes, ctypes.byref(opts), _stream(stream)),
           "lpar_allreduce_f32")


def lpar_status_string(status):
    return _lib.lpar_status_string(status).decode()


def lpar_host_staging_bytes(N, chunk, codec):
    return _lib.lpar_host_staging_bytes(N, chunk, _codec(codec))


def lpar_host_staging_bytes_f32(N, chunk, codec):
    return _lib.lpar_host_staging_bytes_f32(N, chunk, _codec(codec))


def lpar_allreduce_f32_host(host_inputs, n, codec, host_out, chunk, device, device_bytes, min_quant_bytes=0,
                            schedule="auto", stream=None, N=None, stage_events=None):
    """All-reduce of N binary32 messages in host memory, chunk by chunk through
    `device` staging of lpar_host_staging_bytes_f32 bytes."""
    ins = _ptr_array(host_inputs, _host_ptr)
    outs = _ptr_array(host_out, _host_ptr)
    N = len(host_inputs) if N is None else N
    opts = _options(min_quant_bytes, schedule, stage_events)
    _check(_lib.lpar_allreduce_f32_host(ins, N, n, _codec(codec), outs,
                                        chunk, _ptr(device), device_bytes, ctypes.byref(opts), _stream(stream)),
           "lpar_allreduce_f32_host")


def lpar_allreduce_host(host_inputs, n, codec, host_out, chunk, device, device_bytes, min_quant_bytes=0,
                        schedule="auto", stream=None, N=None, stage_events=None):
    """All-reduce of N messages in host memory (pinned for overlap), chunk by
    chunk through `device` staging of lpar_host_staging_bytes bytes."""
    ins = _ptr_array(host_inputs, _host_ptr)
    outs = _ptr_array(host_out, _host_ptr)
    N = len(host_inputs) if N is None else N
    opts = _options(min_quant_bytes, schedule, stage_events)
    _check(_lib.lpar_allreduce_host(ins, N, n, _codec(codec), outs, chunk,
                                    _ptr(device), device_bytes, ctypes.byref(opts), _stream(stream)),
           "lpar_allreduce_host")


def lpar_peer_mailbox_bytes(N, n, codec):
    return _lib.lpar_peer_mailbox_bytes(N, n, _codec(codec))


def lpar_peer_gather_bytes(n, codec):
    return _lib.lpar_peer_gather_bytes(n, _codec(codec))


def lpar_peer_flag_bytes(N, n):
    return _lib.lpar_peer_flag_bytes(N, n)


def _addr(x):
    """Address of a tensor (device or host) or a raw integer address."""
    if x is None or isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("lpar: tensors must be contiguous")
    return x.data_ptr()


def lpar_allreduce_peer(inputs, outputs, mailboxes, gathered, flags, n, codec, timeout_ns, status, rank0=0,
                        ranks=None, stream=None):
    """inputs/outputs: N entries (None outside the launch's ranks); mailboxes,
    gathered, flags: N buffers (tensors or addresses, on this GPU or reachable
    from it); status: LPAR_PEER_STATUS_WORDS words of this GPU's memory (word 4
    carries the epoch from call to call)."""
    N = len(mailboxes)
    ranks = N - rank0 if ranks is None else ranks
    _check(_lib.lpar_allreduce_peer(_ptr_array(inputs, _addr), _ptr_array(outputs, _addr),
                                    _ptr_array(mailboxes, _addr), _ptr_array(gathered, _addr),
                                    _ptr_array(flags, _addr), N, rank0, ranks, n, _codec(codec), int(timeout_ns),
                                    _ptr(status), _stream(stream)), "lpar_allreduce_peer")


def lpar_peer_alloc(nbytes):
    """Device address of `nbytes` of zeroed, IPC-exportable memory."""
    p = ctypes.c_void_p()
    _check(_lib.lpar_peer_alloc(nbytes, ctypes.byref(p)), "lpar_peer_alloc")
    return p.value


def lpar_peer_free(ptr):
    _check(_lib.lpar_peer_free(ptr), "lpar_peer_free")


def lpar_peer_export(ptr):
    """The IPC handle of an lpar_peer_alloc'd address, as bytes."""
    h = ctypes.create_string_buffer(LPAR_PEER_HANDLE_BYTES)
    _check(_lib.lpar_peer_export(ptr, h), "lpar_peer_export")
    return h.raw


def lpar_peer_import(handle):
    """Map another process's lpar_peer_alloc'd memory; returns its address here."""
    if len(handle) != LPAR_PEER_HANDLE_BYTES:
        raise ValueError("lpar: an IPC handle has %d bytes" % LPAR_PEER_HANDLE_BYTES)
    p = ctypes.c_void_p()
    _check(_lib.lpar_peer_import(handle, ctypes.byref(p)), "lpar_peer_import")
    return p.value


def lpar_peer_close(ptr):
    _check(_lib.lpar_peer_close(ptr), "lpar_peer_close")


def lpar_collective_workspace_bytes(op, N, size, codec):
    return _lib.lpar_collective_workspace_bytes(OPS[op] if isinstance(op, str) else int(op), N, size, _codec(codec))


def _collective(fn, name, inputs, size, codec, out, workspace, workspace_bytes, min_quant_bytes, stream, N,
                stage_events):
    ins = _ptr_array(inputs)
    outs = _ptr_array(out)
    N = len(inputs) if N is None else N
    opts = _options(min_quant_bytes, "auto", stage_events)
    _check(fn(ins, N, size, _codec(codec), outs, _ptr(workspace),
              workspace_bytes, ctypes.byref(opts), _stream(stream)), name)


def lpar_reduce_scatter(inputs, n, codec, out, workspace, workspace_bytes, min_quant_bytes=0, stream=None, N=None,
                        stage_events=None):
    _collective(_lib.lpar_reduce_scatter, "lpar_reduce_scatter", inputs, n, codec, out, workspace, workspace_bytes,
                min_quant_bytes, stream, N, stage_events)


def lpar_all_gather(inputs, m, codec, out, workspace, workspace_bytes, min_quant_bytes=0, stream=None, N=None,
                    stage_events=None):
    _collective(_lib.lpar_all_gather, "lpar_all_gather", inputs, m, codec, out, workspace, workspace_bytes,
                min_quant_bytes, stream, N, stage_events)


def lpar_all_to_all(inputs, m, codec, out, workspace, workspace_bytes, min_quant_bytes=0, stream=None, N=None,
                    stage_events=None):
    _collective(_lib.lpar_all_to_all, "lpar_all_to_all", inputs, m, codec, out, workspace, workspace_bytes,
                min_quant_bytes, stream, N, stage_events)


# ---- convenience: allocate with torch, then call the C ABI -----------------------
def allreduce(inputs, codec, out=None, workspace=None, min_quant_bytes=0, schedule="auto", stream=None):
    """All-reduce a list of N equal-size BF16 CUDA tensors; returns the N outputs."""
    import torch
    n = inputs[0].numel()
    if out is None:
        out = [torch.empty_like(x) for x in inputs]
    need = lpar_workspace_bytes(len(inputs), n, lpar_effective_codec(n, codec, min_quant_bytes))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=inputs[0].device)
    lpar_allreduce(inputs, n, codec, out, workspace, workspace.numel(), min_quant_bytes, schedule, stream)
    return out


HOST_CHUNK_ELEMS = 8 << 20          # 16 MiB of BF16 per rank per chunk


def allreduce_host(host_inputs, codec, out=None, chunk=HOST_CHUNK_ELEMS, device_buffer=None, min_quant_bytes=0,
                   schedule="auto", stream=None, device=None):
    """All-reduce a list of N equal-size BF16 host tensors (pin them for overlap)
    through the device in chunks; returns the N host outputs (pinned when
    allocated here).  The result equals `allreduce` of the same values."""
    import torch
    n = host_inputs[0].numel()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = [torch.empty(n, dtype=torch.bfloat16, pin_memory=True) for _ in host_inputs]
    c = max(2048, min(chunk, n))
    need = lpar_host_staging_bytes(len(host_inputs), c, lpar_effective_codec(n, codec, min_quant_bytes))
    if device_buffer is None:
        device_buffer = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    lpar_allreduce_host(host_inputs, n, codec, out, c, device_buffer, device_buffer.numel(), min_quant_bytes,
                        schedule, stream)
    return out


def allreduce_f32_host(host_inputs, codec, out=None, chunk=HOST_CHUNK_ELEMS // 2, device_buffer=None,
                       min_quant_bytes=0, stream=None, device=None):
    """All-reduce a list of N equal-size binary32 host tensors (pin them for
    overlap) through the device in chunks; returns the N host outputs."""
    import torch
    n = host_inputs[0].numel()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = [torch.empty(n, dtype=torch.float32, pin_memory=True) for _ in host_inputs]
    c = max(2048, min(chunk, n))
    need = lpar_host_staging_bytes_f32(len(host_inputs), c, lpar_effective_codec(2 * n, codec, min_quant_bytes))
    if device_buffer is None:
        device_buffer = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    lpar_allreduce_f32_host(host_inputs, n, codec, out, c, device_buffer, device_buffer.numel(), min_quant_bytes,
                            "auto", stream)
    return out


def shard_tiles(N, T):
    """Tile range [t0, t1) of reduce-scatter shard j, j = 0..N-1 (floor partition)."""
    return [(j * T // N, (j + 1) * T // N) for j in range(N)]


def _workspace(op, N, size, codec, min_quant_bytes, device):
    import torch
    n_msg = N * size if op == "all_to_all" else size
    need = lpar_collective_workspace_bytes(op, N, size, lpar_effective_codec(n_msg, codec, min_quant_bytes))
    return torch.empty(max(need, 16), dtype=torch.uint8, device=device)


def reduce_scatter(inputs, codec, min_quant_bytes=0, stream=None):
    """Reduce-scatter of N equal-size BF16 CUDA tensors; returns the N shards."""
    import torch
    N, n = len(inputs), inputs[0].numel()
    out = [torch.empty(max((t1 - t0) * TILE_ELEMS, 8), dtype=torch.bfloat16, device=inputs[0].device)
           for t0, t1 in shard_tiles(N, n // TILE_ELEMS)]
    ws = _workspace("reduce_scatter", N, n, codec, min_quant_bytes, inputs[0].device)
    lpar_reduce_scatter(inputs, n, codec, out, ws, ws.numel(), min_quant_bytes, stream)
    return [o[:(t1 - t0) * TILE_ELEMS] for o, (t0, t1) in zip(out, shard_tiles(N, n // TILE_ELEMS))]


def all_gather(inputs, codec, min_quant_bytes=0, stream=None):
    """All-gather of N BF16 CUDA tensors of m elements; returns N tensors of N * m."""
    import torch
    N, m = len(inputs), inputs[0].numel()
    out = [torch.empty(N * m, dtype=torch.bfloat16, device=inputs[0].device) for _ in range(N)]
    ws = _workspace("all_gather", N, m, codec, min_quant_bytes, inputs[0].device)
    lpar_all_gather(inputs, m, codec, out, ws, ws.numel(), min_quant_bytes, stream)
    return out


def all_to_all(inputs, codec, min_quant_bytes=0, stream=None):
    """All-to-all of N BF16 CUDA tensors of N * m elements (N segments of m)."""
    import torch
    N = len(inputs)
    m = inputs[0].numel() // N
    out = [torch.empty(N * m, dtype=torch.bfloat16, device=inputs[0].device) for _ in range(N)]
    ws = _workspace("all_to_all", N, m, codec, min_quant_bytes, inputs[0].device)
    lpar_all_to_all(inputs, m, codec, out, ws, ws.numel(), min_quant_bytes, stream)
    return out


class PeerTimeout(RuntimeError):
    """A wait of lpar_allreduce_peer gave up: (phase, waiting rank, flag index)."""


class PeerBuffers:
    """The buffers of lpar_allreduce_peer for N ranks that all live on one GPU
    (mailboxes, gathered wires and flags as torch tensors, zeroed) and the
    status words.  One set serves any number of calls of the same (N, n,
    codec) in stream order, CUDA graph replays included."""

    def __init__(self, N, n, codec, device=None):
        import torch
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.N, self.n, self.codec = N, n, codec
        u8 = dict(dtype=torch.uint8, device=dev)
        self.mailboxes = [torch.zeros(max(lpar_peer_mailbox_bytes(N, n, codec), 16), **u8) for _ in range(N)]
        self.gathered = [torch.zeros(max(lpar_peer_gather_bytes(n, codec), 16), **u8) for _ in range(N)]
        self.flags = [torch.zeros(max(lpar_peer_flag_bytes(N, n), 16), **u8) for _ in range(N)]
        self.status = torch.zeros(LPAR_PEER_STATUS_WORDS, dtype=torch.int32, device=dev)

    def allreduce(self, inputs, out, timeout_ns=1_000_000_000, stream=None):
        lpar_allreduce_peer(inputs, out, self.mailboxes, self.gathered, self.flags, self.n, self.codec, timeout_ns,
                            self.status, 0, self.N, stream)
        return out

    def epoch(self):
        """Synchronise and return the epoch of the last call."""
        return int(self.status[4].item()) & 0xFFFFFFFF

    def check(self):
        """Synchronise and raise PeerTimeout if a wait gave up."""
        w = [int(v) for v in self.status.cpu()]
        if w[0]:
            raise PeerTimeout("lpar_allreduce_peer: a wait gave up (phase %d, rank %d, flag %d)" % tuple(w[1:4]))


def allreduce_peer(inputs, codec, out=None, buffers=None, timeout_ns=1_000_000_000, stream=None):
    """All-reduce of N equal-size BF16 CUDA tensors by the peer-memory kernel,
    all ranks in one launch on this GPU; returns the N outputs (equal to
    `allreduce`'s).  Pass `buffers` (a PeerBuffers) to reuse them across calls."""
    import torch
    N, n = len(inputs), inputs[0].numel()
    if out is None:
        out = [torch.empty_like(x) for x in inputs]
    if buffers is None:
        buffers = PeerBuffers(N, n, codec, inputs[0].device)
    return buffers.allreduce(inputs, out, timeout_ns, stream)


def allreduce_f32(inputs, codec, out=None, min_quant_bytes=0, stream=None):
    """All-reduce a list of N equal-size binary32 CUDA tensors; returns the N outputs."""
    import torch
    N, n = len(inputs), inputs[0].numel()
    if out is None:
        out = [torch.empty_like(x) for x in inputs]
    eff = lpar_effective_codec(2 * n, codec, min_quant_bytes)      # threshold on 4n bytes
    need = lpar_collective_workspace_bytes("allreduce_f32", N, n, eff)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=inputs[0].device)
    lpar_allreduce_f32(inputs, n, codec, out, ws, ws.numel(), min_quant_bytes, "auto", stream)
    return out
