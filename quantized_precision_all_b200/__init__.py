"""B200-native compressed all-reduce (INT4 / INT3 / FP8 / MXFP4 / BF16 codecs) behind a C ABI.

The compute lives in ``liblpar.so`` (hand-written sm_100a CUDA kernels, see
``csrc/``); :mod:`.lpar` is the ctypes binding with the C function names.
Build the library with ``python quantized_precision_all_b200/build.py``.
"""
from .lpar import (CODECS, LparError, all_gather, all_to_all, allreduce, allreduce_f32,  # noqa: F401
                   allreduce_f32_host, allreduce_host, lpar_all_gather, lpar_all_to_all, lpar_allreduce, lpar_allreduce_f32,
                   lpar_allreduce_f32_host, lpar_allreduce_host, lpar_allreduce_static, lpar_collective_workspace_bytes, lpar_decode,
                   lpar_effective_codec, lpar_host_staging_bytes, lpar_host_staging_bytes_f32, lpar_quantize, lpar_reduce, lpar_reduce_scatter,
                   lpar_status_string, lpar_tile_bytes, lpar_wire_bytes, lpar_workspace_bytes, reduce_scatter,
                   PeerBuffers, PeerTimeout, allreduce_peer, lpar_allreduce_peer, lpar_peer_alloc, lpar_peer_close,
                   lpar_peer_export, lpar_peer_flag_bytes, lpar_peer_free, lpar_peer_gather_bytes, lpar_peer_import,
                   lpar_peer_mailbox_bytes)
