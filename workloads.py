"""Seeded synthetic inputs for the compressed all-reduce (shared by tests and bench).

This module holds no arithmetic of the method itself: it only draws seeded
random BF16 activations of the shapes and distributions of the workloads and
names those workloads.  Both the CUDA path and the CPU oracle consume its output.

Recipe (rank r of a workload with seed S): a ``torch.Generator`` on the chosen
device seeded with ``S * 1009 + r`` draws binary32 values, which are rounded to
BF16 (round to nearest even) by ``Tensor.to(torch.bfloat16)`` (binary32
workloads keep the draws).
Distributions:
  * ``normal``            N(0, sigma^2)
  * ``normal_outliers``   N(0, 1), then round(0.1% * n) positions per rank,
                          drawn without replacement, multiplied by 50
  * ``student_t``         Z / sqrt(C / nu), C a sum of nu squared N(0,1) draws
"""
from dataclasses import dataclass
from typing import List, Optional, Tuple

import torch

TILE_ELEMS = 2048


@dataclass(frozen=True)
class Workload:
    name: str
    N: int                      # simulated ranks
    n: int                      # BF16 elements per rank
    dist: str                   # normal | normal_outliers | student_t
    seed: int
    codecs: Tuple[str, ...]     # codecs run back to back in one step
    sigma: float = 1.0
    nu: int = 4
    min_quant_bytes: int = 0
    shape: Optional[Tuple[int, ...]] = None
    note: str = ""
    dtype: str = "bf16"         # message element type: bf16, or f32 (binary32 messages)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def message_bytes(self) -> int:
        return self.elem_bytes * self.n


# The workloads of the pages' problem statement (TP activations of LLM serving).
WORKLOADS = {
    "small_int4": Workload(
        "small_int4", N=2, n=65536, dist="normal", seed=1, codecs=("int4",),
        note="N=2 x 65,536 BF16 (128 KiB per rank), N(0,1), INT4"),
    "decode_int3": Workload(
        "decode_int3", N=2, n=64 * 8192, dist="normal_outliers", seed=2, codecs=("int3",),
        min_quant_bytes=1 << 20, shape=(64, 8192),
        note="decode-shaped: N=2 x (64 tokens x 8192 hidden) BF16 = 1 MiB per rank, "
             "N(0,1) with 0.1% outliers x50, INT3 with a 1 MiB activation threshold"),
    "prefill_fp8": Workload(
        "prefill_fp8", N=8, n=2048 * 8192, dist="student_t", nu=4, seed=3, codecs=("fp8", "bf16"),
        shape=(2048, 8192),
        note="prefill-shaped: N=8 x (2048 tokens x 8192 hidden) BF16 = 32 MiB per rank, "
             "Student-t nu=4, FP8 e4m3 and the uncompressed BF16 sum"),
    "large_int3_int4": Workload(
        "large_int3_int4", N=2, n=512 * 1024 * 1024, dist="normal", sigma=0.02, seed=4,
        codecs=("int3", "int4"),
        note="large message: N=2 x 512 Mi BF16 (1 GiB per rank), N(0, 0.02^2), "
             "INT3 then INT4 back to back"),
}

WORKLOADS["prefill_fp8_f32"] = Workload(
    "prefill_fp8_f32", N=8, n=2048 * 8192, dist="student_t", nu=4, seed=3, codecs=("fp8", "bf16"),
    shape=(2048, 8192), dtype="f32",
    note="prefill-shaped, binary32 messages: N=8 x (2048 tokens x 8192 hidden) FP32 = 64 MiB per rank, "
         "Student-t nu=4, FP8 e4m3 (4:1 against FP32) and the uncompressed FP32 sum")
WORKLOADS["large_mxfp4"] = Workload(
    "large_mxfp4", N=2, n=512 * 1024 * 1024, dist="normal", sigma=0.02, seed=4, codecs=("mxfp4",),
    note="large message, FP4 mode: N=2 x 512 Mi BF16 (1 GiB per rank), N(0, 0.02^2), MXFP4")

# A smaller case of the large workload for ncu captures: inputs (256 MiB) still
# exceed the 126 MB L2, while the whole footprint stays under 1 GiB.
PROFILE_WORKLOADS = {
    "profile_int3_int4": Workload(
        "profile_int3_int4", N=2, n=64 * 1024 * 1024, dist="normal", sigma=0.02, seed=4,
        codecs=("int3", "int4"),
        note="profiling case: N=2 x 64 Mi BF16 (128 MiB per rank), N(0, 0.02^2), INT3 then INT4"),
}
WORKLOADS.update(PROFILE_WORKLOADS)

SWEEP_SIZES_BYTES = [1 << k for k in range(17, 31)]    # 128 KiB ... 1 GiB per rank
SWEEP_RANKS = (2, 4, 8)
SWEEP_CODECS = ("bf16", "fp8", "int4", "int3", "mxfp4")


def sweep_workload(N: int, message_bytes: int, codec: str) -> Workload:
    return Workload(f"sweep_N{N}_{message_bytes}B_{codec}", N=N, n=message_bytes // 2,
                    dist="student_t", nu=3, seed=5, codecs=(codec,))


def _draw_f32(w: Workload, r: int, n: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1009 + r)
    if w.dist == "normal":
        return torch.randn(n, generator=g, device=device, dtype=torch.float32) * w.sigma
    if w.dist == "normal_outliers":
        x = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        k = int(round(0.001 * n))
        if k:
            pos = torch.randperm(n, generator=g, device=device)[:k]
            x[pos] *= 50.0
        return x
    if w.dist == "student_t":
        z = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        c = torch.zeros(n, device=device, dtype=torch.float32)
        for _ in range(w.nu):
            y = torch.randn(n, generator=g, device=device, dtype=torch.float32)
            c += y * y
        return z / torch.sqrt(c / w.nu)
    raise ValueError(f"unknown distribution {w.dist!r}")


def make_inputs(w: Workload, device="cpu", n: Optional[int] = None) -> List[torch.Tensor]:
    """N tensors of n elements each (default: the workload's n): BF16, or the
    binary32 draws themselves for an f32 workload."""
    n = w.n if n is None else n
    if w.dtype == "f32":
        return [_draw_f32(w, r, n, device) for r in range(w.N)]
    return [_draw_f32(w, r, n, device).to(torch.bfloat16) for r in range(w.N)]


def make_rank_input(w: Workload, r: int, device="cpu", n: Optional[int] = None) -> torch.Tensor:
    """Rank r's message alone (the same values as ``make_inputs(w)[r]``; r may
    exceed w.N when the ranks are real processes)."""
    n = w.n if n is None else n
    x = _draw_f32(w, r, n, device)
    return x if w.dtype == "f32" else x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """BF16 tensor -> numpy uint16 bit patterns on the host."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
