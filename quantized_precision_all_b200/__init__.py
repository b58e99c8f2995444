"""B200-native compressed all-reduce (INT4 / INT3 / FP8 / BF16 codecs) behind a C ABI.

The compute lives in ``liblpar.so`` (hand-written sm_100a CUDA kernels, see
``csrc/``); :mod:`.lpar` is the ctypes binding with the C function names.
Build the library with ``python -m quantized_precision_all_b200.build``.
"""
from .lpar import (CODECS, LparError, allreduce, lpar_allreduce, lpar_decode, lpar_effective_codec,  # noqa: F401
                   lpar_quantize, lpar_reduce, lpar_status_string, lpar_tile_bytes, lpar_wire_bytes,
                   lpar_workspace_bytes)
