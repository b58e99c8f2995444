"""ctypes view of the CPU oracle (``lpar_oracle.c``).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It never touches the CUDA library.

Arrays are numpy: BF16 data travels as ``uint16`` bit patterns, wires as
``uint8``.  Codecs are named by string: ``bf16``, ``fp8``, ``int4``, ``int3``,
``mxfp4``.
"""
import ctypes
import os

import numpy as np

from . import build_oracle

CODECS = {"bf16": 0, "fp8": 1, "int4": 2, "int3": 3, "mxfp4": 4}
TILE_ELEMS = 2048
BLOCK = 32
MAX_RANKS = 8

_lib = None


def lib():
    global _lib
    if _lib is None:
        # A test may point this at another build of the same source.
        path = os.environ.get("LPAR_ORACLE_LIB") or build_oracle.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        sz = ctypes.c_size_t
        sig = {
            "orc_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
            "orc_f32_to_bf16_rne": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f32_to_f16_rne": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
            "orc_e4m3_to_f32": (ctypes.c_float, [ctypes.c_uint8]),
            "orc_f32_to_e4m3_rne_satfinite": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_e2m1_to_f32": (ctypes.c_float, [ctypes.c_uint8]),
            "orc_e2m1_rne_satfinite": (ctypes.c_uint8, [ctypes.c_double]),
            "orc_e8m0_to_f64": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_tile_bytes": (sz, [ctypes.c_int]),
            "orc_wire_bytes": (sz, [ctypes.c_int, sz]),
            "orc_quant_block_int": (None, [f32p, ctypes.c_int, u16p, u8p]),
            "orc_dequant_int": (ctypes.c_float, [ctypes.c_uint8, ctypes.c_int, ctypes.c_uint16]),
            "orc_quant_block_fp8": (None, [f32p, f32p, u8p]),
            "orc_dequant_fp8": (ctypes.c_float, [ctypes.c_uint8, ctypes.c_float]),
            "orc_quant_block_mxfp4": (None, [f32p, u8p, u8p]),
            "orc_dequant_mxfp4": (ctypes.c_float, [ctypes.c_uint8, ctypes.c_uint8]),
            "orc_quant_tile": (None, [f32p, ctypes.c_int, u8p]),
            "orc_tile_code": (ctypes.c_uint8, [u8p, ctypes.c_int, ctypes.c_int]),
            "orc_dequant_tile": (None, [u8p, ctypes.c_int, f32p]),
            "orc_quantize": (None, [u16p, sz, ctypes.c_int, u8p]),
            "orc_reduce": (None, [ctypes.POINTER(u8p), ctypes.c_int, sz, sz, ctypes.c_int, u8p]),
            "orc_decode": (None, [u8p, sz, ctypes.c_int, u16p]),
            "orc_allreduce": (ctypes.c_int, [ctypes.POINTER(u16p), ctypes.c_int, sz, ctypes.c_int,
                                             ctypes.POINTER(u16p), sz]),
            "orc_reduce_scatter": (ctypes.c_int, [ctypes.POINTER(u16p), ctypes.c_int, sz, ctypes.c_int,
                                                  ctypes.POINTER(u16p), sz]),
            "orc_allreduce_oneshot": (ctypes.c_int, [ctypes.POINTER(u16p), ctypes.c_int, sz, ctypes.c_int,
                                                     ctypes.POINTER(u16p), sz]),
            "orc_all_gather": (ctypes.c_int, [ctypes.POINTER(u16p), ctypes.c_int, sz, ctypes.c_int,
                                              ctypes.POINTER(u16p), sz]),
            "orc_all_to_all": (ctypes.c_int, [ctypes.POINTER(u16p), ctypes.c_int, sz, ctypes.c_int,
                                              ctypes.POINTER(u16p), sz]),
            "orc_allreduce_f32": (ctypes.c_int, [ctypes.POINTER(f32p), ctypes.c_int, sz, ctypes.c_int,
                                                 ctypes.POINTER(f32p), sz]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _codec(codec):
    return CODECS[codec] if isinstance(codec, str) else int(codec)


# ---- scalar conversions ----------------------------------------------------
def bf16_to_f32(h):
    return lib().orc_bf16_to_f32(int(h))


def f32_to_bf16(x):
    return lib().orc_f32_to_bf16_rne(float(np.float32(x)))


def f32_to_f16(x):
    return lib().orc_f32_to_f16_rne(float(np.float32(x)))


def f16_to_f32(h):
    return lib().orc_f16_to_f32(int(h))


def e4m3_to_f32(e):
    return lib().orc_e4m3_to_f32(int(e))


def f32_to_e4m3(x):
    return lib().orc_f32_to_e4m3_rne_satfinite(float(np.float32(x)))


def e2m1_to_f32(c):
    return lib().orc_e2m1_to_f32(int(c))


def e2m1_rne(y):
    """A real value (Python float, binary64) -> E2M1 code."""
    return lib().orc_e2m1_rne_satfinite(float(y))


def e8m0_value(code):
    return lib().orc_e8m0_to_f64(int(code))


# ---- geometry --------------------------------------------------------------
def tile_bytes(codec):
    return lib().orc_tile_bytes(_codec(codec))


def wire_bytes(codec, n):
    return lib().orc_wire_bytes(_codec(codec), n)


# ---- blocks and tiles ------------------------------------------------------
def quant_block_int(x, bits):
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == BLOCK
    sb = ctypes.c_uint16()
    codes = np.zeros(BLOCK, np.uint8)
    lib().orc_quant_block_int(_ptr(x, ctypes.c_float), bits, ctypes.byref(sb), _ptr(codes, ctypes.c_uint8))
    return sb.value, codes


def dequant_int(code, bits, scale_bits):
    return lib().orc_dequant_int(int(code), bits, int(scale_bits))


def quant_block_fp8(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == BLOCK
    s = ctypes.c_float()
    codes = np.zeros(BLOCK, np.uint8)
    lib().orc_quant_block_fp8(_ptr(x, ctypes.c_float), ctypes.byref(s), _ptr(codes, ctypes.c_uint8))
    return s.value, codes


def dequant_fp8(code, scale):
    return lib().orc_dequant_fp8(int(code), float(np.float32(scale)))


def quant_block_mxfp4(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == BLOCK
    sc = ctypes.c_uint8()
    codes = np.zeros(BLOCK, np.uint8)
    lib().orc_quant_block_mxfp4(_ptr(x, ctypes.c_float), ctypes.byref(sc), _ptr(codes, ctypes.c_uint8))
    return sc.value, codes


def dequant_mxfp4(code, scale_code):
    return lib().orc_dequant_mxfp4(int(code), int(scale_code))


def quant_tile(x, codec):
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == TILE_ELEMS
    tile = np.zeros(tile_bytes(codec), np.uint8)
    lib().orc_quant_tile(_ptr(x, ctypes.c_float), _codec(codec), _ptr(tile, ctypes.c_uint8))
    return tile


def tile_codes(tile, codec):
    tile = np.ascontiguousarray(tile, dtype=np.uint8)
    L = lib()
    p = _ptr(tile, ctypes.c_uint8)
    return np.array([L.orc_tile_code(p, _codec(codec), i) for i in range(TILE_ELEMS)], np.uint8)


def dequant_tile(tile, codec):
    tile = np.ascontiguousarray(tile, dtype=np.uint8)
    v = np.zeros(TILE_ELEMS, np.float32)
    lib().orc_dequant_tile(_ptr(tile, ctypes.c_uint8), _codec(codec), _ptr(v, ctypes.c_float))
    return v


# ---- stages ----------------------------------------------------------------
def quantize(x_bf16, codec):
    """Stage 1: BF16 bit patterns (uint16, n % 2048 == 0) -> wire bytes."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1)
    wire = np.zeros(wire_bytes(codec, x.size), np.uint8)
    lib().orc_quantize(_ptr(x, ctypes.c_uint16), x.size, _codec(codec), _ptr(wire, ctypes.c_uint8))
    return wire


def reduce(wires, tile_begin, tile_count, codec, wire_out=None):
    """Stage 2 over tiles [tile_begin, tile_begin+tile_count) of full wires."""
    wires = [np.ascontiguousarray(w, dtype=np.uint8) for w in wires]
    if wire_out is None:
        wire_out = np.zeros_like(wires[0])
    arr = (ctypes.POINTER(ctypes.c_uint8) * len(wires))(*[_ptr(w, ctypes.c_uint8) for w in wires])
    lib().orc_reduce(arr, len(wires), tile_begin, tile_count, _codec(codec), _ptr(wire_out, ctypes.c_uint8))
    return wire_out


def decode(wire, n, codec):
    """Stage 3: wire -> BF16 bit patterns (uint16)."""
    wire = np.ascontiguousarray(wire, dtype=np.uint8)
    out = np.zeros(n, np.uint16)
    lib().orc_decode(_ptr(wire, ctypes.c_uint8), n, _codec(codec), _ptr(out, ctypes.c_uint16))
    return out


def allreduce(inputs_bf16, codec, min_quant_bytes=0):
    """Whole collective over N host arrays of BF16 bits; returns (outputs, codec used)."""
    ins = [np.ascontiguousarray(x, dtype=np.uint16).reshape(-1) for x in inputs_bf16]
    n = ins[0].size
    outs = [np.zeros(n, np.uint16) for _ in ins]
    ia = (ctypes.POINTER(ctypes.c_uint16) * len(ins))(*[_ptr(x, ctypes.c_uint16) for x in ins])
    oa = (ctypes.POINTER(ctypes.c_uint16) * len(outs))(*[_ptr(o, ctypes.c_uint16) for o in outs])
    used = lib().orc_allreduce(ia, len(ins), n, _codec(codec), oa, min_quant_bytes)
    if used < 0:
        raise ValueError("oracle rejected the arguments")
    name = {v: k for k, v in CODECS.items()}[used]
    return outs, name


def bf16_bits_to_f32(bits):
    """Vectorised exact widening of BF16 bit patterns (numpy, no rounding)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _collective(fn, inputs_bf16, codec, out_sizes, size_arg, min_quant_bytes):
    ins = [np.ascontiguousarray(x, dtype=np.uint16).reshape(-1) for x in inputs_bf16]
    outs = [np.zeros(k, np.uint16) for k in out_sizes]
    ia = (ctypes.POINTER(ctypes.c_uint16) * len(ins))(*[_ptr(x, ctypes.c_uint16) for x in ins])
    oa = (ctypes.POINTER(ctypes.c_uint16) * len(outs))(*[_ptr(o, ctypes.c_uint16) for o in outs])
    used = fn(ia, len(ins), size_arg, _codec(codec), oa, min_quant_bytes)
    if used < 0:
        raise ValueError("oracle rejected the arguments")
    return outs, {v: k for k, v in CODECS.items()}[used]


def shard_tiles(N, T):
    """Tile range [t0, t1) of shard j for j = 0..N-1 (floor partition)."""
    return [(j * T // N, (j + 1) * T // N) for j in range(N)]


def reduce_scatter(inputs_bf16, codec, min_quant_bytes=0):
    """Rank j gets its shard of the BF16 sum; returns (outputs, codec used)."""
    n = np.asarray(inputs_bf16[0]).size
    sizes = [(t1 - t0) * TILE_ELEMS for t0, t1 in shard_tiles(len(inputs_bf16), n // TILE_ELEMS)]
    return _collective(lib().orc_reduce_scatter, inputs_bf16, codec, sizes, n, min_quant_bytes)


def allreduce_oneshot(inputs_bf16, codec, min_quant_bytes=0):
    n = np.asarray(inputs_bf16[0]).size
    return _collective(lib().orc_allreduce_oneshot, inputs_bf16, codec, [n] * len(inputs_bf16), n,
                       min_quant_bytes)


def all_gather(inputs_bf16, codec, min_quant_bytes=0):
    """Each of N ranks contributes m elements; every rank gets all N * m."""
    N, m = len(inputs_bf16), np.asarray(inputs_bf16[0]).size
    return _collective(lib().orc_all_gather, inputs_bf16, codec, [N * m] * N, m, min_quant_bytes)


def all_to_all(inputs_bf16, codec, min_quant_bytes=0):
    """Each rank's N * m elements are N segments of m, segment j bound for rank j."""
    N = len(inputs_bf16)
    m = np.asarray(inputs_bf16[0]).size // N
    return _collective(lib().orc_all_to_all, inputs_bf16, codec, [N * m] * N, m, min_quant_bytes)


def allreduce_f32(inputs_f32, codec, min_quant_bytes=0):
    """All-reduce of N binary32 host arrays; returns (binary32 outputs, codec used)."""
    ins = [np.ascontiguousarray(x, dtype=np.float32).reshape(-1) for x in inputs_f32]
    n = ins[0].size
    outs = [np.zeros(n, np.float32) for _ in ins]
    fp = ctypes.POINTER(ctypes.c_float)
    ia = (fp * len(ins))(*[_ptr(x, ctypes.c_float) for x in ins])
    oa = (fp * len(outs))(*[_ptr(o, ctypes.c_float) for o in outs])
    used = lib().orc_allreduce_f32(ia, len(ins), n, _codec(codec), oa, min_quant_bytes)
    if used < 0:
        raise ValueError("oracle rejected the arguments")
    return outs, {v: k for k, v in CODECS.items()}[used]
