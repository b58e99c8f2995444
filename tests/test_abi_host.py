"""The C-ABI library on the host: it loads without a GPU, exports every symbol
the header declares, reports the page-fixed sizes, and rejects bad arguments
before launching anything (no GPU is touched by any call here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lpar.h")


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\w[\w\s\*]*?\b(lpar_\w+)\s*\(", text, re.M)))


def test_header_is_valid_c():
    subprocess.run(["gcc", "-std=c11", "-fsyntax-only", "-Wall", "-Werror", "-x", "c",
                    "-I", "/usr/local/cuda/include", HEADER], check=True)


def test_library_exports_every_declared_symbol(L):
    decl = declared_functions()
    assert decl, "no declarations parsed"
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (lpar_\w+)", out))
    assert set(decl) <= exported, set(decl) - exported
    assert set(L.EXPORTS) == set(decl)
    for name in decl:
        assert hasattr(L.library(), name)


def test_tile_and_wire_sizes(L):
    assert L.lpar_tile_bytes("int4") == 1152
    assert L.lpar_tile_bytes("int3") == 896
    assert L.lpar_tile_bytes("fp8") == 2304
    assert L.lpar_tile_bytes("bf16") == 4096
    assert L.lpar_tile_bytes("mxfp4") == 1088
    assert L.lpar_tile_bytes(7) == 0
    assert L.lpar_wire_bytes("int3", 2048 * 3) == 3 * 896
    assert L.lpar_wire_bytes("int4", 2048 * 5 + 100) == 5 * 1152
    n = 512 * 1024 * 1024
    assert L.lpar_wire_bytes("int3", n) == 234881024 and L.lpar_wire_bytes("int4", n) == 301989888


def test_workspace_bytes(L):
    n = 2048 * 10
    assert L.lpar_workspace_bytes(2, n, "int4") == 3 * 10 * 1152
    assert L.lpar_workspace_bytes(8, n, "fp8") == 9 * 10 * 2304
    assert L.lpar_workspace_bytes(2, n, "int3") == 3 * 10 * 896
    assert L.lpar_workspace_bytes(4, n, "bf16") == 2 * n
    assert L.lpar_workspace_bytes(3, n, "mxfp4") == 4 * 10 * 1088
    assert L.lpar_workspace_bytes(0, n, "int4") == 0
    assert L.lpar_workspace_bytes(9, n, "int4") == 0


def test_effective_codec_threshold(L):
    thr = 1 << 20
    assert L.lpar_effective_codec(thr // 2, "int3", thr) == "int3"          # 1 MiB message: >= threshold
    assert L.lpar_effective_codec(thr // 2 - 2048, "int3", thr) == "bf16"
    assert L.lpar_effective_codec(2048, "fp8", 0) == "fp8"
    assert L.lpar_effective_codec(2048, "bf16", thr) == "bf16"


# Fake, never-dereferenced device addresses: every call below must fail in
# validation before any launch.
A = 0x7F0000000000          # 16-byte aligned
M = A + 8                   # misaligned


def status_of(fn, *args, **kw):
    from quantized_precision_all_b200.lpar import LparError
    try:
        fn(*args, **kw)
    except LparError as e:
        return e.status
    return 0


def test_argument_errors_quantize(L):
    st = 0
    assert status_of(L.lpar_quantize, A, 2048, 9, A, st) == 4            # unknown codec
    assert status_of(L.lpar_quantize, A, 2047, "int4", A, st) == 1       # n not a tile multiple
    assert status_of(L.lpar_quantize, 0, 2048, "int4", A, st) == 1       # null input
    assert status_of(L.lpar_quantize, A, 2048, "int4", 0, st) == 1       # null wire
    assert status_of(L.lpar_quantize, M, 2048, "int4", A, st) == 2       # misaligned
    assert status_of(L.lpar_quantize, A, 2048, "int3", M, st) == 2
    assert status_of(L.lpar_quantize, 0, 0, "int4", 0, st) == 0          # empty message: no-op
    assert status_of(L.lpar_quantize, A, 2048 * (2 ** 33 + 1), "int4", A, st) == 1   # beyond 2^44


def test_argument_errors_reduce_decode(L):
    st = 0
    assert status_of(L.lpar_reduce, [A] * 9, 0, 1, "int4", A, st) == 1   # N > 8
    assert status_of(L.lpar_reduce, [A, 0], 0, 1, "int4", A, st) == 1    # null wire
    assert status_of(L.lpar_reduce, [A, M], 0, 1, "int4", A, st) == 2
    assert status_of(L.lpar_reduce, [A, A], 0, 1, "int4", M, st) == 2
    assert status_of(L.lpar_reduce, [A, A], 0, 1, 5, A, st) == 4
    assert status_of(L.lpar_reduce, [A, A], 2 ** 64 - 1, 2, "int4", A, st) == 1   # range overflow
    assert status_of(L.lpar_reduce, [A, A], 3, 0, "int4", A, st) == 0    # empty range: no-op
    assert status_of(L.lpar_decode, A, 100, "int4", A, st) == 1
    assert status_of(L.lpar_decode, A, 2048, "fp8", M, st) == 2
    assert status_of(L.lpar_decode, 0, 2048, "fp8", A, st) == 1


def test_argument_errors_allreduce(L):
    st = 0
    n = 2048 * 4
    ws = L.lpar_workspace_bytes(2, n, "int4")
    ok = dict(min_quant_bytes=0, schedule="auto", stream=st)
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, A], A, ws - 16, **ok) == 3
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, M], A, ws, **ok) == 2
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, A], M, ws, **ok) == 2
    assert status_of(L.lpar_allreduce, [A, 0], n, "int4", [A, A], A, ws, **ok) == 1
    assert status_of(L.lpar_allreduce, [A, A], n + 1, "int4", [A, A], A, ws, **ok) == 1
    assert status_of(L.lpar_allreduce, [A] * 9, n, "int4", [A] * 9, A, 10 ** 9, **ok) == 1
    assert status_of(L.lpar_allreduce, [A, A], n, 11, [A, A], A, ws, **ok) == 4
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, A], A, ws, min_quant_bytes=0, schedule=7,
                     stream=st) == 4
    assert status_of(L.lpar_allreduce, [A, A], 0, "int4", [A, A], A, 0, **ok) == 0
    # raw C call with null arrays
    lib = L.library()
    opts = L.lpar_options_t(0, 0)
    assert lib.lpar_allreduce(None, 2, n, 2, None, A, ws, ctypes.byref(opts), None) == 1
    assert lib.lpar_allreduce(None, 2, n, 2, None, A, ws, None, None) == 1


def test_collective_workspace_bytes(L):
    n = 2048 * 10
    assert L.lpar_collective_workspace_bytes("allreduce", 2, n, "int4") == L.lpar_workspace_bytes(2, n, "int4")
    assert L.lpar_collective_workspace_bytes("reduce_scatter", 3, n, "int3") == 3 * 10 * 896
    assert L.lpar_collective_workspace_bytes("all_gather", 4, n, "mxfp4") == 4 * 10 * 1088
    assert L.lpar_collective_workspace_bytes("all_to_all", 2, n, "fp8") == 2 * 20 * 2304
    for op in ("reduce_scatter", "all_gather", "all_to_all"):
        assert L.lpar_collective_workspace_bytes(op, 2, n, "bf16") == 0
        assert L.lpar_collective_workspace_bytes(op, 9, n, "int4") == 0
        assert L.lpar_collective_workspace_bytes(op, 2, n, 9) == 0
    assert L.lpar_collective_workspace_bytes(7, 2, n, "int4") == 0


@pytest.mark.parametrize("fn", ["lpar_reduce_scatter", "lpar_all_gather", "lpar_all_to_all"])
def test_argument_errors_collectives(L, fn):
    call = getattr(L, fn)
    op = fn[len("lpar_"):]
    st = 0
    n = 2048 * 4
    ws = L.lpar_collective_workspace_bytes(op, 2, n, "int4")
    assert status_of(call, [A, A], n, "int4", [A, A], A, ws - 16, stream=st) == 3
    assert status_of(call, [A, A], n, "int4", [A, M], A, ws, stream=st) == 2
    assert status_of(call, [M, A], n, "int4", [A, A], A, ws, stream=st) == 2
    assert status_of(call, [A, A], n, "int4", [A, A], M, ws, stream=st) == 2
    assert status_of(call, [A, 0], n, "int4", [A, A], A, ws, stream=st) == 1
    assert status_of(call, [A, A], n, "int4", [A, A], 0, ws, stream=st) == 1      # workspace needed
    assert status_of(call, [A, A], n + 1, "int4", [A, A], A, ws, stream=st) == 1
    assert status_of(call, [A] * 9, n, "int4", [A] * 9, A, 10 ** 9, stream=st) == 1
    assert status_of(call, [A, A], n, 11, [A, A], A, ws, stream=st) == 4
    assert status_of(call, [A, A], 0, "int4", [A, A], 0, 0, stream=st) == 0       # empty: no-op
    big = 2048 * (2 ** 33 + 1)
    assert status_of(call, [A, A], big, "int4", [A, A], A, 10 ** 18, stream=st) == 1
    assert status_of(call, [A] * 4, 2 ** 62, "int4", [A] * 4, A, 10 ** 18, stream=st) == 1   # 4 * 2^62 wraps
    if op == "all_to_all":                                   # N * m above 2^44 although m is not
        assert status_of(call, [A] * 4, 2 ** 43, "int4", [A] * 4, A, 2 ** 62, stream=st) == 1
    lib = L.library()
    opts = L.lpar_options_t(0, 0)
    assert getattr(lib, fn)(None, 2, n, 2, None, A, ws, ctypes.byref(opts), None) == 1


def test_argument_errors_allreduce_f32(L):
    st = 0
    n = 2048 * 4
    need = L.lpar_collective_workspace_bytes("allreduce_f32", 2, n, "fp8")
    assert need == 3 * 4 * 2304
    assert L.lpar_collective_workspace_bytes("allreduce_f32", 2, n, "bf16") == 4 * n
    ok = dict(stream=st)
    assert status_of(L.lpar_allreduce_f32, [A, A], n, "fp8", [A, A], A, need - 16, **ok) == 3
    assert status_of(L.lpar_allreduce_f32, [A, M], n, "fp8", [A, A], A, need, **ok) == 2
    assert status_of(L.lpar_allreduce_f32, [A, A], n, "fp8", [A, A], M, need, **ok) == 2
    assert status_of(L.lpar_allreduce_f32, [A, A], n, "fp8", [A, A], 0, need, **ok) == 1
    assert status_of(L.lpar_allreduce_f32, [A, A], n + 4, "fp8", [A, A], A, need, **ok) == 1
    assert status_of(L.lpar_allreduce_f32, [A] * 9, n, "fp8", [A] * 9, A, 10 ** 9, **ok) == 1
    assert status_of(L.lpar_allreduce_f32, [A, A], n, 12, [A, A], A, need, **ok) == 4
    assert status_of(L.lpar_allreduce_f32, [A, A], n, "fp8", [A, A], A, need, schedule="fused", **ok) == 4
    assert status_of(L.lpar_allreduce_f32, [A, A], 0, "fp8", [A, A], A, 0, **ok) == 0


def test_one_shot_schedule_is_accepted_and_validated(L):
    st = 0
    n = 2048 * 4
    ws = L.lpar_workspace_bytes(2, n, "int4")
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, A], A, ws - 16, schedule="one_shot", stream=st) == 3
    assert status_of(L.lpar_allreduce, [A, A], n, "int4", [A, A], A, ws, schedule=5, stream=st) == 4


def test_host_staging_bytes(L):
    c = 2048 * 8
    assert L.lpar_host_staging_bytes(2, c, "int3") == 3 * 2 * 2 * c + L.lpar_workspace_bytes(2, c, "int3")
    assert L.lpar_host_staging_bytes(8, c, "bf16") == 3 * 8 * 2 * c + L.lpar_workspace_bytes(8, c, "bf16")
    assert L.lpar_host_staging_bytes(0, c, "int4") == 0
    assert L.lpar_host_staging_bytes(9, c, "int4") == 0
    assert L.lpar_host_staging_bytes(2, 0, "int4") == 0
    assert L.lpar_host_staging_bytes(2, c + 4, "int4") == 0
    assert L.lpar_host_staging_bytes(2, c, 11) == 0


def test_argument_errors_allreduce_host(L):
    # host "addresses" are never touched: every call fails in validation first
    H = 0x10000
    n, c = 2048 * 6, 2048 * 4
    need = L.lpar_host_staging_bytes(2, c, "int4")
    f = L.lpar_allreduce_host
    assert status_of(f, [H, H], n, "int4", [H, H], c, A, need - 16, stream=0) == 3
    assert status_of(f, [H, H], n, "int4", [H, H], c, M, need, stream=0) == 2
    assert status_of(f, [H, H], n, "int4", [H, H], c, 0, need, stream=0) == 1
    assert status_of(f, [H, 0], n, "int4", [H, H], c, A, need, stream=0) == 1
    assert status_of(f, [H, H], n + 2, "int4", [H, H], c, A, need, stream=0) == 1
    assert status_of(f, [H, H], n, "int4", [H, H], c + 2, A, need, stream=0) == 1
    assert status_of(f, [H, H], n, "int4", [H, H], 0, A, need, stream=0) == 1
    assert status_of(f, [H] * 9, n, "int4", [H] * 9, c, A, 10 ** 9, stream=0) == 1
    assert status_of(f, [H, H], n, 12, [H, H], c, A, need, stream=0) == 4
    assert status_of(f, [H, H], n, "int4", [H, H], c, A, need, schedule=5, stream=0) == 4
    assert status_of(f, [H, H], 0, "int4", [H, H], c, A, 0, stream=0) == 0
    # a chunk larger than the message is the message: staging for n suffices
    small = L.lpar_host_staging_bytes(2, n, "int4")
    assert status_of(f, [H, H], n, "int4", [H, H], 2048 * 64, A, small - 16, stream=0) == 3


def test_host_staging_bytes_f32(L):
    c = 2048 * 8
    assert L.lpar_host_staging_bytes_f32(8, c, "fp8") == 3 * 8 * 4 * c + \
        L.lpar_collective_workspace_bytes("allreduce_f32", 8, c, "fp8")
    assert L.lpar_host_staging_bytes_f32(2, c, "bf16") == 3 * 2 * 4 * c + 4 * c
    assert L.lpar_host_staging_bytes_f32(0, c, "fp8") == 0
    assert L.lpar_host_staging_bytes_f32(2, c + 2, "fp8") == 0


def test_argument_errors_allreduce_f32_host(L):
    H = 0x10000
    n, c = 2048 * 6, 2048 * 4
    need = L.lpar_host_staging_bytes_f32(2, c, "fp8")
    f = L.lpar_allreduce_f32_host
    assert status_of(f, [H, H], n, "fp8", [H, H], c, A, need - 16, stream=0) == 3
    assert status_of(f, [H, H], n, "fp8", [H, H], c, M, need, stream=0) == 2
    assert status_of(f, [H, 0], n, "fp8", [H, H], c, A, need, stream=0) == 1
    assert status_of(f, [H, H], n + 2, "fp8", [H, H], c, A, need, stream=0) == 1
    assert status_of(f, [H, H], n, 12, [H, H], c, A, need, stream=0) == 4
    assert status_of(f, [H, H], n, "fp8", [H, H], c, A, need, schedule="fused", stream=0) == 4
    assert status_of(f, [H, H], 0, "fp8", [H, H], c, A, 0, stream=0) == 0


def test_status_strings(L):
    for s in range(6):
        assert L.lpar_status_string(s)
    assert "unknown" in L.lpar_status_string(99)


def test_python_binding_rejects_host_tensors(L):
    import torch
    x = torch.zeros(2048, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        L.lpar_quantize(x, 2048, "int4", x)


def test_peer_buffer_bytes(L):
    n = 2048 * 10
    assert L.lpar_peer_mailbox_bytes(3, n, "int4") == 3 * 4 * 1152        # 3 slots of ceil(10 / 3) tiles
    assert L.lpar_peer_mailbox_bytes(2, n, "bf16") == 2 * 5 * 4096
    assert L.lpar_peer_mailbox_bytes(1, n, "mxfp4") == 10 * 1088
    assert L.lpar_peer_gather_bytes(n, "int3") == 10 * 896
    assert L.lpar_peer_gather_bytes(n, "fp8") == 10 * 2304
    # chunks of about N T / 592 tiles (1 to 16, a multiple of 4 above 4), at most 1024 per shard
    assert L.lpar_peer_flag_bytes(3, n) == 2 * 3 * 4 * 4                  # 1-tile chunks: P = ceil(10 / 3)
    assert L.lpar_peer_flag_bytes(8, 2048 << 20) == 2 * 8 * 1024 * 4      # P capped at 1024
    assert L.lpar_peer_flag_bytes(8, 2048 * 8 * 1024) == 2 * 8 * 64 * 4  # 16-tile chunks
    assert L.lpar_peer_flag_bytes(8, 2048 * (8 * 16 * 1000 + 1)) == 2 * 8 * 1001 * 4
    assert L.lpar_peer_flag_bytes(2, 2048 * 256) == 2 * 2 * 128 * 4       # 1 MiB per rank: 1-tile chunks
    assert L.lpar_peer_flag_bytes(8, 2048 * 256) == 2 * 8 * 8 * 4         # N T / 592 = 3.5: 4-tile chunks
    assert L.lpar_peer_flag_bytes(2, 2048 * 4096) == 2 * 2 * 128 * 4      # 13.8 rounds to 16-tile chunks
    for bad in (L.lpar_peer_mailbox_bytes(0, n, "int4"), L.lpar_peer_mailbox_bytes(9, n, "int4"),
                L.lpar_peer_mailbox_bytes(2, n + 1, "int4"), L.lpar_peer_mailbox_bytes(2, n, 7),
                L.lpar_peer_gather_bytes(n + 2, "int4"), L.lpar_peer_gather_bytes(n, 9),
                L.lpar_peer_flag_bytes(0, n), L.lpar_peer_flag_bytes(2, n + 4), L.lpar_peer_flag_bytes(2, 0)):
        assert bad == 0


def test_argument_errors_allreduce_peer(L):
    n = 2048 * 4

    def call(inputs=(A, A), outputs=(A, A), mailboxes=(A, A), gathered=(A, A), flags=(A, A), n=n, codec="int4",
             timeout_ns=10 ** 6, status=A, rank0=0, ranks=None):
        return status_of(L.lpar_allreduce_peer, list(inputs), list(outputs), list(mailboxes), list(gathered),
                         list(flags), n, codec, timeout_ns, status, rank0=rank0, ranks=ranks, stream=0)

    assert call(timeout_ns=0) == 1
    assert call(status=0) == 1
    assert call(status=M) == 2
    assert call(mailboxes=(A, M)) == 2
    assert call(gathered=(M, A)) == 2
    assert call(flags=(A, 0)) == 1
    assert call(inputs=(A, 0)) == 1                      # rank 1 runs in this launch: it needs an input
    assert call(outputs=(M, A)) == 2
    assert call(n=n + 2048 // 2) == 1
    assert call(codec=9) == 4
    assert call(rank0=1, ranks=2) == 1
    assert call(rank0=-1, ranks=1) == 1
    assert call(ranks=0) == 1
    assert call(inputs=[A] * 9, outputs=[A] * 9, mailboxes=[A] * 9, gathered=[A] * 9, flags=[A] * 9) == 1
    assert call(n=0) == 0                                # a no-op, nothing launched
    assert call(inputs=(A, None), outputs=(A, None), ranks=1, n=0) == 0   # rank 1 outside: no input needed
    lib = L.library()
    assert lib.lpar_allreduce_peer(None, None, None, None, None, 2, 0, 2, n, 2, 10, A, None) == 1


def test_peer_ipc_argument_errors(L):
    lib = L.library()
    assert lib.lpar_peer_alloc(0, None) == 1
    assert lib.lpar_peer_free(None) == 1
    assert lib.lpar_peer_export(None, None) == 1
    assert lib.lpar_peer_import(None, None) == 1
    assert lib.lpar_peer_close(None) == 1
    with pytest.raises(ValueError):
        L.lpar_peer_import(b"\0" * 10)


def test_peer_sizes_fit_the_chunk_geometry(L):
    """For many (N, T): the library's flag count gives P chunks per shard, of
    1 to 16 tiles by the message size, at most 1024; the
    chunks [cS/P, (c+1)S/P) tile every shard exactly; a mailbox slot holds the
    largest shard; the gathered wire holds every tile."""
    for N in range(1, 9):
        for T in list(range(1, 70)) + [127, 128, 129, 1023, 1025, 4099, 16 * 1024 * 8 + 5, 1 << 20]:
            n = T * 2048
            P = L.lpar_peer_flag_bytes(N, n) // (2 * N * 4)
            smax = -(-T // N)
            ct = min(max(-(-(N * T) // 592), 1), 16)
            ct = -(-ct // 4) * 4 if ct > 4 else ct
            assert 1 <= P <= 1024 and P == min(max(-(-smax // ct), 1), 1024), (N, T, P)
            tb = L.lpar_tile_bytes("int4")
            assert L.lpar_peer_mailbox_bytes(N, n, "int4") == N * smax * tb
            assert L.lpar_peer_gather_bytes(n, "int4") == T * tb
            if T > 5000:
                continue                                   # the partition check below is O(N P)
            covered = 0
            for j in range(N):
                base, S = j * T // N, (j + 1) * T // N - j * T // N
                assert S <= smax
                prev = base
                for c in range(P):
                    lo, hi = base + c * S // P, base + (c + 1) * S // P
                    assert lo == prev and lo <= hi
                    prev = hi
                    covered += hi - lo
                assert prev == base + S
            assert covered == T


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the Python package without liblpar.so: importing the binding (or the
    cross-process module built on it) raises OSError -- there is no fallback path."""
    import shutil
    import sys
    pkg = tmp_path / "quantized_precision_all_b200"
    pkg.mkdir()
    for f in ("__init__.py", "lpar.py", "distributed.py"):
        shutil.copy(os.path.join(ROOT, "quantized_precision_all_b200", f), pkg / f)
    for mod in ("quantized_precision_all_b200.lpar", "quantized_precision_all_b200.distributed"):
        r = subprocess.run([sys.executable, "-c", "import %s" % mod], cwd=tmp_path, capture_output=True, text=True,
                           env={**os.environ, "PYTHONPATH": str(tmp_path)})
        assert r.returncode != 0 and "OSError" in r.stderr, (mod, r.stderr[-500:])
