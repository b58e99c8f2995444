"""The all-reduce of binary32 messages on the GPU against the CPU oracle, bit for
bit (needs a B200).  Inputs are seeded binary32 blocks of several kinds: wide
ranges of scale, zeros and negative zeros, exact and one-ulp-off ties of the
INT grids at full 24-bit precision, E4M3 and E2M1 grid points and midpoints,
subnormal values.  Guard bands around every buffer the library writes.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.test_gpu_parity import Guarded

pytestmark = pytest.mark.gpu

CODECS = ("int4", "int3", "fp8", "mxfp4", "bf16")


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


def adversarial_f32(n, seed):
    rng = np.random.default_rng(seed)
    x = np.zeros((n // 32, 32), np.float32)
    kinds = rng.integers(0, 8, n // 32)
    for b in range(n // 32):
        k = kinds[b]
        if k == 0:
            x[b] = rng.standard_normal(32) * 10.0 ** rng.uniform(-6, 6)
        elif k == 1:
            x[b] = -0.0
            x[b, rng.integers(32)] = rng.standard_normal()
        elif k in (2, 3):
            # 24-bit values on and next to the INT ties: s = f16(absmax / qmax)
            qmax = 7 if k == 2 else 3
            a = np.float32(rng.uniform(1, 2) * 2.0 ** rng.integers(-8, 8))
            s = np.float32(O.f16_to_f32(O.f32_to_f16(a / np.float32(qmax))))
            q = rng.integers(-qmax, qmax, 32) + 0.5
            v = (q * s).astype(np.float32)
            nudge = rng.integers(-1, 2, 32)
            v = np.where(nudge < 0, np.nextafter(v, -np.inf), np.where(nudge > 0, np.nextafter(v, np.inf), v))
            x[b] = v
            x[b, 0] = a
        elif k == 4:
            e = rng.integers(-30, 30)
            grid = np.array([0, 0.5, 1, 1.5, 2, 2.25, 2.5, 3, 17, 18, 19, 240, 416, 432, 440, 448], np.float32)
            x[b] = rng.choice(grid, 32) * rng.choice([-1, 1], 32) * np.float32(2.0 ** e)
        elif k == 5:
            e = rng.integers(-30, 30)
            grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.75, 2.5, 3.5, 5, 6, 7], np.float32)
            x[b] = rng.choice(grid, 32) * rng.choice([-1, 1], 32) * np.float32(2.0 ** e)
            x[b, 0] = np.float32(rng.choice([4.0, 6.0, 7.5]) * 2.0 ** e)
        elif k == 6:
            x[b] = (rng.standard_normal(32) * 1e-39).astype(np.float32)    # subnormal values
            x[b, 0] = np.float32(rng.choice([1e-38, 3e-39, 1e-30]))
        else:
            x[b] = rng.standard_t(3, 32) * 10.0 ** rng.uniform(20, 33)
    return x.reshape(-1)


def f32_to_device(x):
    g = Guarded(x.size * 4)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(x).view(np.uint8)))
    return g


def run(L, xs, codec, min_quant_bytes=0, inplace=False):
    N, n = len(xs), xs[0].size
    ins = [f32_to_device(x) for x in xs]
    outs = ins if inplace else [Guarded(4 * n, fill=0x00) for _ in range(N)]
    eff = L.lpar_effective_codec(2 * n, codec, min_quant_bytes)
    ws = Guarded(L.lpar_collective_workspace_bytes("allreduce_f32", N, n, eff))
    L.lpar_allreduce_f32([g.ptr() for g in ins], n, codec, [g.ptr() for g in outs], ws.ptr(), ws.nbytes,
                         min_quant_bytes=min_quant_bytes)
    torch.cuda.synchronize()
    for g in outs + [ws] + ([] if inplace else ins):
        g.check()
    return [g.host().view(np.float32) for g in outs], eff


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N,tiles", [(1, 5), (2, 9), (3, 6), (8, 7)])
def test_allreduce_f32_matches_oracle(L, codec, N, tiles):
    n = tiles * 2048
    xs = [adversarial_f32(n, 700 + 10 * N + r) for r in range(N)]
    outs, eff = run(L, xs, codec)
    ref, used = O.allreduce_f32(xs, codec)
    assert eff == used == codec
    for o in outs:
        assert np.array_equal(o.view(np.uint32), ref[0].view(np.uint32))


@pytest.mark.parametrize("codec", ["int3", "fp8"])
def test_allreduce_f32_in_place(L, codec):
    xs = [adversarial_f32(2048 * 5, 800 + r) for r in range(2)]
    outs, _ = run(L, xs, codec, inplace=True)
    ref, _ = O.allreduce_f32(xs, codec)
    for o in outs:
        assert np.array_equal(o.view(np.uint32), ref[0].view(np.uint32))


def test_allreduce_f32_threshold(L):
    thr = 1 << 20
    n = thr // 4 - 2048                              # 4n just below 1 MiB
    xs = [adversarial_f32(n, 900 + r) for r in range(2)]
    outs, eff = run(L, xs, "fp8", min_quant_bytes=thr)
    ref, used = O.allreduce_f32(xs, "fp8", thr)
    assert eff == used == "bf16"
    assert np.array_equal(outs[0].view(np.uint32), ref[0].view(np.uint32))


def test_allreduce_f32_prefill_shape_sampled(L):
    """N = 8 x (2048 x 8192) binary32 (64 MiB per rank), FP8, Student-t: the
    RCCLX case of FP8 against FP32 inputs; 256 seeded random tiles plus the
    first and last are compared (tiles are independent)."""
    N, n = 8, 2048 * 8192
    g = torch.Generator(device="cuda")
    xs = []
    for r in range(N):
        g.manual_seed(3 * 1009 + r)
        z = torch.randn(n, generator=g, device="cuda")
        c = sum(torch.randn(n, generator=g, device="cuda") ** 2 for _ in range(4))
        xs.append((z / torch.sqrt(c / 4)).contiguous())
    outs = L.allreduce_f32(xs, "fp8")
    torch.cuda.synchronize()
    T = n // 2048
    rng = np.random.default_rng(10)
    tiles = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 256, replace=False)]))
    idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
    sample = [x[idx].cpu().numpy() for x in xs]
    ref, _ = O.allreduce_f32(sample, "fp8")
    for o in outs:
        assert np.array_equal(o[idx].cpu().numpy().view(np.uint32), ref[0].view(np.uint32))


# Seeded random cases: codec, N in 1..8, 1..30 tiles, a threshold either side
# of the binary32 message, in place or not.
@pytest.mark.parametrize("case", range(24))
def test_allreduce_f32_random_cases(L, case):
    rng = np.random.default_rng(9700 + case)
    codec = CODECS[rng.integers(len(CODECS))]
    N = int(rng.integers(1, 9))
    tiles = int(rng.integers(1, 31))
    n = tiles * 2048
    thr = (0, 4 * n, 4 * n + 4)[rng.integers(3)]
    inplace = bool(rng.integers(2))
    xs = [adversarial_f32(n, int(rng.integers(1 << 20))) for _ in range(N)]
    outs, eff = run(L, xs, codec, min_quant_bytes=thr, inplace=inplace)
    ref, used = O.allreduce_f32(xs, codec, thr)
    assert eff == used
    for o in outs:
        assert np.array_equal(o.view(np.uint32), ref[0].view(np.uint32)), (codec, N, tiles, thr, inplace)

