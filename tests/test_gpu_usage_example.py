"""A short usage example of the Python binding, run on the GPU: the calls a
user makes first (the all-reduce with and without a caller workspace, the
reduce-scatter, the all-gather, host-resident messages, the peer-memory
kernel), with the results
compared bit for bit with the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def test_usage_example():
    from quantized_precision_all_b200 import lpar as L

    torch.manual_seed(0)
    N, n = 2, 64 * 8192                                   # ranks, BF16 elements per rank (multiple of 2048)
    xs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(N)]
    outs = L.allreduce(xs, "int3", min_quant_bytes=1 << 20)   # every outs[r] holds the same reduced tensor
    torch.cuda.synchronize()
    bits = [_bits(x) for x in xs]
    ref3, used = O.allreduce(bits, "int3", min_quant_bytes=1 << 20)
    assert used == "int3"
    assert all(np.array_equal(_bits(o), ref3[0]) for o in outs)

    # the same with a caller-owned workspace, on an explicit stream
    ws = torch.empty(L.lpar_workspace_bytes(N, n, "fp8"), dtype=torch.uint8, device="cuda")
    L.lpar_allreduce(xs, n, "fp8", outs, ws, ws.numel(), stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    ref8, _ = O.allreduce(bits, "fp8")
    assert all(np.array_equal(_bits(o), ref8[0]) for o in outs)

    rs = L.reduce_scatter(xs, "int4")                        # rank j gets shard j of the sum
    ag = L.all_gather([x[:2048 * 4] for x in xs], "mxfp4")   # every rank gets every rank's block
    host = L.allreduce_host([x.cpu().pin_memory() for x in xs], "int4")   # host tensors in and out
    torch.cuda.synchronize()
    ref_rs, _ = O.reduce_scatter(bits, "int4")
    assert all(np.array_equal(_bits(a), b) for a, b in zip(rs, ref_rs))
    ref_ag, _ = O.all_gather([b[:2048 * 4] for b in bits], "mxfp4")
    assert all(np.array_equal(_bits(a), b) for a, b in zip(ag, ref_ag))
    ref4, _ = O.allreduce(bits, "int4")
    assert all(np.array_equal(h.view(torch.int16).numpy().view(np.uint16), ref4[0]) for h in host)

    # the peer-memory kernel, every rank in one launch; its buffers kept for later calls
    pb = L.PeerBuffers(N, n, "int4")
    peer = L.allreduce_peer(xs, "int4", buffers=pb)
    pb.check()                                               # raises if a wait for a rank gave up
    assert all(np.array_equal(_bits(o), ref4[0]) for o in peer)
