"""lpar_allreduce_static: the all-reduce for callers that cannot allocate device
memory (for example a plugin whose host application owns all device memory),
using the workspace the library keeps for itself.

Its results must equal those of lpar_allreduce with a caller-provided workspace,
on two calls in a row (the shared workspace keeps the previous call's contents),
and once a first call has run on the device, later calls must leave the
device's free memory unchanged.
This file is named to be collected last, and must pass both alone in a fresh
process and after the other tests.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


@pytest.mark.parametrize("codec,N", [("int3", 2), ("int4", 2), ("fp8", 8), ("mxfp4", 4), ("bf16", 3)])
def test_static_workspace_equals_caller_workspace_on_two_calls(L, codec, N):
    n = 2048 * 37
    g = torch.Generator(device="cuda").manual_seed(900 + N)
    ref_out = None
    for call in range(2):
        xs = [(torch.randn(n, generator=g, device="cuda") * 10.0 ** (r - 1)).to(torch.bfloat16) for r in range(N)]
        ws = torch.empty(L.lpar_workspace_bytes(N, n, codec), dtype=torch.uint8, device="cuda")
        ref_out = [torch.empty_like(x) for x in xs]
        L.lpar_allreduce(xs, n, codec, ref_out, ws, ws.numel())
        out = [torch.full_like(x, float("nan")) for x in xs]
        L.lpar_allreduce_static(xs, n, codec, out)
        torch.cuda.synchronize()
        for o, r in zip(out, ref_out):
            assert torch.equal(o.view(torch.int16), r.view(torch.int16)), (codec, call)


def test_static_calls_allocate_nothing(L):
    N, n = 4, 2048 * 200
    xs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(N)]
    out = [torch.empty_like(x) for x in xs]
    L.lpar_allreduce_static(xs, n, "int4", out)          # the first call may load the library's module
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for codec in ("int4", "int3", "fp8", "mxfp4", "bf16", "int4"):
        L.lpar_allreduce_static(xs, n, codec, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_static_workspace_rejects_messages_beyond_its_size(L):
    n = 2048 * 4096                                   # INT3, N = 2: 3 * 3.5 MiB fits
    xs = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    out = [torch.empty_like(x) for x in xs]
    L.lpar_allreduce_static(xs, n, "int3", out)
    big = L.LPAR_STATIC_WORKSPACE_BYTES // 2 + 2048    # BF16 needs 2n bytes > the array
    ys = [torch.zeros(big - big % 2048 + 2048, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(L.LparError) as e:
        L.lpar_allreduce_static(ys, ys[0].numel(), "bf16", [torch.empty_like(y) for y in ys])
    assert e.value.status == 3
    torch.cuda.synchronize()
