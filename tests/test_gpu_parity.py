"""CUDA path vs the CPU oracle, element by element (needs a B200).

Every comparison is bit-exact: wires (codes + scales) byte for byte and BF16
outputs bit for bit -- the path is deterministic and follows the same
definitions, so the 1-ulp BF16 allowance is not needed.  Inputs are seeded and
synthetic; expected values come only from the oracle.  Every device buffer the
library writes has 4 KiB guard bands on both sides, checked after each call.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5
CODECS = ("int4", "int3", "fp8", "mxfp4", "bf16")
QCODECS = ("int4", "int3", "fp8", "mxfp4")


@pytest.fixture(scope="module")
def L():
    from quantized_precision_all_b200 import build
    build.build()
    from quantized_precision_all_b200 import lpar
    return lpar


class Guarded:
    """A device byte buffer with canary bands on both sides."""

    def __init__(self, nbytes, fill=CANARY):
        self.nbytes = nbytes
        self.buf = torch.full((nbytes + 2 * GUARD,), fill, dtype=torch.uint8, device="cuda")
        self.buf[:GUARD] = CANARY
        self.buf[GUARD + nbytes:] = CANARY

    @property
    def t(self):
        return self.buf[GUARD:GUARD + self.nbytes]

    def ptr(self):
        return self.buf.data_ptr() + GUARD          # also valid (and aligned) for an empty region

    def host(self):
        return self.t.cpu().numpy()

    def check(self):
        assert torch.all(self.buf[:GUARD] == CANARY), "front guard overwritten"
        assert torch.all(self.buf[GUARD + self.nbytes:] == CANARY), "back guard overwritten"


def to_device(bits_u16):
    g = Guarded(bits_u16.size * 2)
    g.t.copy_(torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.uint8)))
    return g


def host_u16(g):
    return g.host().view(np.uint16)


def f16_value(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


# ---------------------------------------------------------------------------
# Adversarial BF16 inputs (seeded): block kinds cycle through random normal at
# random scales, all-zero, single outliers, exact ties of the INT grids,
# saturating magnitudes, tiny magnitudes (subnormal scales), negative zeros,
# E4M3 and E2M1 grid points, midpoints and saturation.
# ---------------------------------------------------------------------------
def bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def adversarial_bf16(n, seed):
    rng = np.random.default_rng(seed)
    nb = n // 32
    x = np.zeros((nb, 32), np.float32)
    kinds = rng.integers(0, 10, nb)
    for b in range(nb):
        k = kinds[b]
        if k == 0:
            x[b] = rng.standard_normal(32) * 10.0 ** rng.uniform(-4, 4)
        elif k == 1:
            pass                                                     # all zero
        elif k == 2:
            x[b] = rng.standard_normal(32) * 0.01
            x[b, rng.integers(32)] = rng.choice([-1, 1]) * 10.0 ** rng.uniform(0, 6)
        elif k in (3, 4):
            # on-grid block with ties: s = m * 2^e with a 3-bit m keeps (k + 1/2) s in BF16
            qmax = 7 if k == 3 else 3
            s = rng.choice([1.0, 1.25, 1.5, 1.75]) * 2.0 ** rng.integers(-12, 12)
            q = rng.integers(-qmax, qmax, 32) + rng.choice([0.0, 0.5], 32)
            q[rng.integers(32)] = qmax * rng.choice([-1, 1])
            x[b] = q * s
        elif k == 5:
            x[b] = rng.standard_normal(32) * 10.0 ** rng.uniform(5, 37)  # saturating scales
        elif k == 6:
            x[b] = rng.standard_normal(32) * 10.0 ** rng.uniform(-39, -4)  # subnormal / zero scales
        elif k == 7:
            x[b] = -0.0
            x[b, rng.integers(32)] = rng.standard_normal()
        elif k == 9:
            # MXFP4 ties and saturation: E2M1 grid points, midpoints and values in
            # (6, 8) at a power-of-two scale, some with tiny (E8M0-clamped) scales
            e = rng.integers(-20, 20) if rng.random() < 0.8 else rng.integers(-140, -126)
            grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7], np.float32)
            x[b] = rng.choice(grid, 32) * rng.choice([-1, 1], 32) * 2.0 ** e
            x[b, rng.integers(32)] = rng.choice([4.0, 6.0, 7.5]) * 2.0 ** e
        else:
            # FP8 ties and saturation: E4M3 grid points and midpoints at a power-of-two scale
            e = rng.integers(-20, 20)
            grid = np.array([0.0, 0.5, 1, 1.5, 2, 2.25, 2.5, 3, 17, 18, 19, 240, 416, 432, 440, 448], np.float32)
            x[b] = rng.choice(grid, 32) * rng.choice([-1, 1], 32) * 2.0 ** e
            x[b, rng.integers(32)] = 448 * 2.0 ** e
    bits = bf16(x.reshape(-1))
    neg0 = (kinds == 7).repeat(32) & (x.reshape(-1) == 0)
    bits[neg0] = 0x8000
    return bits


def random_bf16(n, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, generator=g) * scale).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# Stage 1
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("tiles", [1, 3, 5, 37])
def test_quantize_matches_oracle(L, codec, tiles):
    n = tiles * 2048
    x = adversarial_bf16(n, seed=1000 + tiles)
    dx = to_device(x)
    wire = Guarded(L.lpar_wire_bytes(codec, n))
    L.lpar_quantize(dx.ptr(), n, codec, wire.ptr())
    torch.cuda.synchronize()
    wire.check()
    dx.check()
    assert np.array_equal(wire.host(), O.quantize(x, codec))


@pytest.mark.parametrize("codec", QCODECS)
def test_quantize_every_bf16_value_as_block_absmax_candidate(L, codec):
    # block p = [bf16 pattern p, 31 fixed values]: every finite BF16 value meets the scale path
    pats = np.array([p for p in range(0x10000) if (p & 0x7F80) != 0x7F80], np.uint16)
    pats = np.concatenate([pats, np.zeros((-len(pats)) % 64, np.uint16)])
    others = random_bf16(31, seed=7, scale=3.0)
    x = np.empty((len(pats), 32), np.uint16)
    x[:, 0] = pats
    x[:, 1:] = others
    x = x.reshape(-1)
    n = x.size
    dx = to_device(x)
    wire = Guarded(L.lpar_wire_bytes(codec, n))
    L.lpar_quantize(dx.ptr(), n, codec, wire.ptr())
    torch.cuda.synchronize()
    wire.check()
    assert np.array_equal(wire.host(), O.quantize(x, codec))


# ---------------------------------------------------------------------------
# Stage 3
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("codec", CODECS)
def test_decode_matches_oracle(L, codec):
    n = 2048 * 11
    wire = O.quantize(adversarial_bf16(n, seed=31), codec)
    dw = Guarded(wire.size)
    dw.t.copy_(torch.from_numpy(wire))
    out = Guarded(2 * n)
    L.lpar_decode(dw.ptr(), n, codec, out.ptr())
    torch.cuda.synchronize()
    out.check()
    assert np.array_equal(host_u16(out), O.decode(wire, n, codec))


@pytest.mark.parametrize("codec", ["int4", "int3", "mxfp4"])
def test_decode_arbitrary_code_bytes(L, codec):
    # any code byte pattern is a valid INT or E2M1 code; keep scales finite
    n = 2048 * 6
    rng = np.random.default_rng(32)
    wire = rng.integers(0, 256, L.lpar_wire_bytes(codec, n), dtype=np.uint8)
    tb = L.lpar_tile_bytes(codec)
    for t in range(n // 2048):
        if codec == "mxfp4":                              # E8M0 bytes 0..254 (255 is NaN)
            wire[t * tb + 1024:t * tb + tb] = rng.integers(0, 255, 64).astype(np.uint8)
            continue
        sc = rng.integers(0, 0x7C00, 64).astype(np.uint16) | (rng.integers(0, 2, 64).astype(np.uint16) << 15)
        wire[t * tb + tb - 128:t * tb + tb] = sc.view(np.uint8)
    dw = Guarded(wire.size)
    dw.t.copy_(torch.from_numpy(wire))
    out = Guarded(2 * n)
    L.lpar_decode(dw.ptr(), n, codec, out.ptr())
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(out), O.decode(wire, n, codec))


# ---------------------------------------------------------------------------
# Stage 2
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
def test_reduce_matches_oracle_on_a_tile_range(L, codec, N):
    tiles = 13
    n = tiles * 2048
    wires = [O.quantize(adversarial_bf16(n, seed=200 + r) if r % 2 else random_bf16(n, 300 + r, 10.0 ** (r - 3)),
                        codec) for r in range(N)]
    dws = []
    for w in wires:
        g = Guarded(w.size)
        g.t.copy_(torch.from_numpy(w))
        dws.append(g)
    out = Guarded(wires[0].size)                      # pre-filled with the canary byte
    t0, cnt = 2, 9                                    # a ragged range: 2 full CTAs + 1 tile
    L.lpar_reduce([g.ptr() for g in dws], t0, cnt, codec, out.ptr())
    torch.cuda.synchronize()
    out.check()
    ref = O.reduce(wires, t0, cnt, codec, wire_out=np.full(wires[0].size, CANARY, np.uint8))
    assert np.array_equal(out.host(), ref)            # tiles outside the range untouched


def arbitrary_wire(codec, n, rng, tile_bytes):
    """Random code bytes (every bit pattern is a code the decoder accepts, including
    the INT codes -2^(b-1) that the encoder never writes) with random scales:
    binary16 of either sign, subnormals and 65504 included; E8M0 bytes 0..249.
    Non-finite values are outside the method's definition, so the E8M0 bytes stop
    where a sum of eight decoded values stays finite (|e| 2^E <= 6 * 2^122)."""
    wire = rng.integers(0, 256, (n // 2048) * tile_bytes, dtype=np.uint8)
    for t in range(n // 2048):
        if codec == "mxfp4":
            wire[t * tile_bytes + 1024:(t + 1) * tile_bytes] = rng.integers(0, 250, 64).astype(np.uint8)
        else:
            sc = rng.integers(0, 0x7C00, 64).astype(np.uint16) | (rng.integers(0, 2, 64).astype(np.uint16) << 15)
            wire[(t + 1) * tile_bytes - 128:(t + 1) * tile_bytes] = sc.view(np.uint8)
    return wire


@pytest.mark.parametrize("codec", ["int4", "int3", "mxfp4"])
@pytest.mark.parametrize("N", [1, 2, 3, 8])
def test_reduce_arbitrary_code_bytes(L, codec, N):
    # stage 2 decodes every code pattern of N ranks, sums and requantises; the
    # sums reach the saturated and subnormal scales
    n = 2048 * 5
    rng = np.random.default_rng(400 + N)
    tb = L.lpar_tile_bytes(codec)
    wires = [arbitrary_wire(codec, n, rng, tb) for _ in range(N)]
    for w in wires:                                   # finite by construction
        assert np.all((O.decode(w, n, codec) & 0x7FFF) < 0x7F80)
    dws = []
    for w in wires:
        g = Guarded(w.size)
        g.t.copy_(torch.from_numpy(w))
        dws.append(g)
    out = Guarded(wires[0].size)
    L.lpar_reduce([g.ptr() for g in dws], 0, n // 2048, codec, out.ptr())
    torch.cuda.synchronize()
    out.check()
    assert np.array_equal(out.host(), O.reduce(wires, 0, n // 2048, codec))


@pytest.mark.parametrize("bits,codec", [(4, "int4"), (3, "int3")])
def test_reduce_exact_ties_at_stage_two(L, bits, codec):
    # rank 0 holds q0 * S (absmax qmax * S), rank 1 holds odd multiples of S/2 with
    # its own absmax qmax * S/2, so every FP32 sum is an exact tie (k + 1/2) S of the
    # requantisation grid while the block absmax stays qmax * S.
    qmax = 2 ** (bits - 1) - 1
    rng = np.random.default_rng(40 + bits)
    n = 2048 * 5
    x0 = np.zeros(n, np.float32)
    x1 = np.zeros(n, np.float32)
    for b in range(n // 32):
        S = rng.choice([1.0, 1.25, 1.5, 1.75]) * 2.0 ** rng.integers(-10, 10)
        q1 = rng.choice(np.arange(-qmax, qmax + 1, 2), 32).astype(np.float32)   # odd multiples
        q0 = rng.integers(-(qmax // 2), qmax // 2 + 1, 32).astype(np.float32)
        q0[0], q1[0] = qmax, 0                          # absmax of the sum: qmax * S
        j = 1 + rng.integers(31)
        q0[j], q1[j] = 0, qmax                          # rank 1's own absmax
        x0[b * 32:(b + 1) * 32] = q0 * S
        x1[b * 32:(b + 1) * 32] = q1 * S / 2
    wires = [O.quantize(bf16(x0), codec), O.quantize(bf16(x1), codec)]
    dws = []
    for w in wires:
        g = Guarded(w.size)
        g.t.copy_(torch.from_numpy(w))
        dws.append(g)
    out = Guarded(wires[0].size)
    L.lpar_reduce([g.ptr() for g in dws], 0, n // 2048, codec, out.ptr())
    torch.cuda.synchronize()
    ref = O.reduce(wires, 0, n // 2048, codec)
    assert np.array_equal(out.host(), ref)
    # the construction really produced ties: sums are odd multiples of S/2
    v = np.concatenate([O.dequant_tile(wires[0][t * len(wires[0]) // 5:(t + 1) * len(wires[0]) // 5], codec)
                        + O.dequant_tile(wires[1][t * len(wires[1]) // 5:(t + 1) * len(wires[1]) // 5], codec)
                        for t in range(5)])
    assert np.count_nonzero(v) > n // 2


@pytest.mark.parametrize("N", [1, 2, 3])
def test_fp8_subnormal_products_and_inputs(L, N):
    # scales near 2^-126 make e4m3(code) * s subnormal; tiny elements next to a
    # normal absmax make x * (1/s) and the FP32 sums subnormal or near it
    rng = np.random.default_rng(77 + N)
    n = 2048 * 3
    xs = []
    for r in range(N):
        x = np.zeros((n // 32, 32), np.float32)
        for b in range(n // 32):
            e = rng.integers(-126, -100) if b % 2 else rng.integers(-20, 5)
            x[b] = rng.standard_normal(32) * 2.0 ** e
            x[b, rng.integers(32)] = 2.0 ** rng.integers(-125, -118) * rng.choice([-1, 1])
            x[b, rng.integers(32)] = rng.choice([1e-39, -1e-39, 3e-40])
        xs.append(bf16(x.reshape(-1)))
    outs, _ = run_allreduce(L, xs, "fp8")
    ref, _ = O.allreduce(xs, "fp8")
    for o in outs:
        assert np.array_equal(o, ref[0])
    wire = O.quantize(xs[0], "fp8")
    dx = to_device(xs[0])
    dw = Guarded(wire.size)
    L.lpar_quantize(dx.ptr(), n, "fp8", dw.ptr())
    torch.cuda.synchronize()
    assert np.array_equal(dw.host(), wire)


@pytest.mark.parametrize("entry", ["reduce", "allreduce"])
def test_mxfp4_stage_two_ties_and_tiny_sums(L, entry):
    # rank 0 sits on the E2M1 grid at 2^E with absmax 6 * 2^E; rank 1 holds
    # 0, +-0.25, +-0.5 times 2^E (its own absmax 0.5 * 2^E, so its grid reaches
    # 0.25 * 2^E).  The sums 0.75, 1.25, 1.75, 2.5, 3.5 (times 2^E) are E2M1
    # midpoints of the requantisation; some blocks use scales near 2^-127 so
    # the dequantised values and sums are subnormal.
    rng = np.random.default_rng(61)
    n = 2048 * 4
    x0 = np.zeros(n, np.float32)
    x1 = np.zeros(n, np.float32)
    g0 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    for b in range(n // 32):
        E = rng.integers(-12, 12) if b % 4 else rng.integers(-128, -121)
        a = rng.choice(g0, 32) * rng.choice([-1, 1], 32)
        c = rng.choice(np.array([0, 0.25, 0.5], np.float32), 32) * rng.choice([-1, 1], 32)
        a[0], c[0] = 6.0, 0.0
        c[1] = 0.5
        x0[b * 32:(b + 1) * 32] = a * 2.0 ** E
        x1[b * 32:(b + 1) * 32] = c * 2.0 ** E
    xs = [bf16(x0), bf16(x1)]
    assert all(np.array_equal(O.bf16_bits_to_f32(b16), x) for b16, x in zip(xs, (x0, x1)))
    if entry == "reduce":
        wires = [O.quantize(x, "mxfp4") for x in xs]
        dws = []
        for w in wires:
            g = Guarded(w.size)
            g.t.copy_(torch.from_numpy(w))
            dws.append(g)
        out = Guarded(wires[0].size)
        L.lpar_reduce([g.ptr() for g in dws], 0, n // 2048, "mxfp4", out.ptr())
        torch.cuda.synchronize()
        assert np.array_equal(out.host(), O.reduce(wires, 0, n // 2048, "mxfp4"))
    else:
        outs, _ = run_allreduce(L, xs, "mxfp4")
        ref, _ = O.allreduce(xs, "mxfp4")
        for o in outs:
            assert np.array_equal(o, ref[0])
    # the construction produced midpoints of the E2M1 grid: a block's sum has
    # absmax in [6, 6.5] * 2^E, so the requantisation divides by 2^E
    sums = (x0 + x1).reshape(-1, 32).astype(np.float64)
    amax = np.max(np.abs(sums), axis=1, keepdims=True)
    scaled = np.abs(sums) / 2.0 ** (np.floor(np.log2(amax)) - 2)
    assert np.count_nonzero(np.isin(scaled, [0.75, 1.25, 1.75, 2.5, 3.5])) > n // 10


@pytest.mark.parametrize("bits,codec", [(4, "int4"), (3, "int3")])
@pytest.mark.parametrize("entry", ["reduce", "allreduce"])
def test_stage_two_near_ties_take_the_exact_path(L, bits, codec, entry):
    # ranks 0 and 1 sit on the grid S/2 (their sum's absmax is qmax * S, so the
    # requantisation scale is S); rank 2 adds q2 * S * 2^-20.  Sums land within
    # 2^-18 of a half-integer multiple of S without being ties, which the fast
    # path must hand to the exact path.
    qmax = 2 ** (bits - 1) - 1
    rng = np.random.default_rng(50 + bits)
    n = 2048 * 3
    xs = [np.zeros(n, np.float32) for _ in range(3)]
    for b in range(n // 32):
        S = 2.0 ** rng.integers(-3, 4)
        q0 = rng.integers(-qmax, qmax + 1, 32).astype(np.float32)
        q1 = rng.integers(-qmax, qmax + 1, 32).astype(np.float32)
        q0[0] = q1[0] = qmax                              # element 0: qmax S, the absmax
        q0[1:] = np.clip(q0[1:], -qmax // 2 - 1, qmax // 2)
        q1[1:] = np.where(np.abs(q0[1:] + q1[1:]) > qmax, 0, q1[1:])
        q2 = rng.integers(-4, 5, 32).astype(np.float32)
        q2[2] = qmax                                      # rank 2's own absmax
        xs[0][b * 32:(b + 1) * 32] = q0 * S / 2
        xs[1][b * 32:(b + 1) * 32] = q1 * S / 2
        xs[2][b * 32:(b + 1) * 32] = q2 * S * 2.0 ** -20
    bits16 = [bf16(x) for x in xs]
    assert all(np.array_equal(O.bf16_bits_to_f32(b16), x) for b16, x in zip(bits16, xs))
    if entry == "reduce":
        wires = [O.quantize(x, codec) for x in bits16]
        dws = []
        for w in wires:
            g = Guarded(w.size)
            g.t.copy_(torch.from_numpy(w))
            dws.append(g)
        out = Guarded(wires[0].size)
        L.lpar_reduce([g.ptr() for g in dws], 0, n // 2048, codec, out.ptr())
        torch.cuda.synchronize()
        assert np.array_equal(out.host(), O.reduce(wires, 0, n // 2048, codec))
    else:
        outs, _ = run_allreduce(L, bits16, codec)
        ref, _ = O.allreduce(bits16, codec)
        for o in outs:
            assert np.array_equal(o, ref[0])


def test_reduce_bf16_rounding_ties(L):
    # 1 + 2^-8 is halfway between two BF16 neighbours; 1 + 3*2^-8 likewise
    n = 2048
    a = np.full(n, 0x3F80, np.uint16)                            # 1.0
    b = bf16(np.where(np.arange(n) % 2 == 0, 2.0 ** -8, 3 * 2.0 ** -8).astype(np.float32))
    wires = [a.view(np.uint8).copy(), b.view(np.uint8).copy()]
    dws = []
    for w in wires:
        g = Guarded(w.size)
        g.t.copy_(torch.from_numpy(w))
        dws.append(g)
    out = Guarded(2 * n)
    L.lpar_reduce([g.ptr() for g in dws], 0, 1, "bf16", out.ptr())
    torch.cuda.synchronize()
    assert np.array_equal(out.host(), O.reduce(wires, 0, 1, "bf16"))


# ---------------------------------------------------------------------------
# The whole all-reduce
# ---------------------------------------------------------------------------
def run_allreduce(L, xs, codec, schedule="auto", min_quant_bytes=0, inplace=False):
    N, n = len(xs), xs[0].size
    ins = [to_device(x) for x in xs]
    outs = ins if inplace else [Guarded(2 * n, fill=0x00) for _ in range(N)]
    ws = Guarded(L.lpar_workspace_bytes(N, n, L.lpar_effective_codec(n, codec, min_quant_bytes)))
    L.lpar_allreduce([g.ptr() for g in ins], n, codec, [g.ptr() for g in outs], ws.ptr(), ws.nbytes,
                     min_quant_bytes=min_quant_bytes, schedule=schedule)
    torch.cuda.synchronize()
    for g in outs + [ws] + ([] if inplace else ins):
        g.check()
    return [host_u16(g) for g in outs], ws


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("N", [1, 2, 3, 8])
@pytest.mark.parametrize("schedule", ["auto", "fused", "three_stage", "single_pass"])
def test_allreduce_matches_oracle(L, codec, N, schedule):
    tiles = 9                                          # 2 CTAs + a ragged one per rank
    n = tiles * 2048
    xs = [adversarial_bf16(n, 500 + r) if r % 2 else random_bf16(n, 600 + r) for r in range(N)]
    outs, ws = run_allreduce(L, xs, codec, schedule)
    ref, used = O.allreduce(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(o, ref[0])
    if codec != "bf16":
        # the workspace holds the stage-1 wires and the gathered wire, as the oracle's
        wb = L.lpar_wire_bytes(codec, n)
        host = ws.host()
        wires = [O.quantize(x, codec) for x in xs]
        for r in range(N):
            assert np.array_equal(host[r * wb:(r + 1) * wb], wires[r])
        assert np.array_equal(host[N * wb:(N + 1) * wb], O.reduce(wires, 0, tiles, codec))


# The single-pass kernel's forms around the limit of the rank-parallel tile
# form (256 tiles per rank, 512 for FP8; one tile per CTA): at and below it
# the tile form, just above it the persistent forms with a ragged last chunk
# (T % 4 == 1 or 3).  Adversarial and random inputs; every output and the
# workspace (stage-1 wires, gathered wire) against the oracle.
def tile_form_limit(codec):
    return 512 if codec == "fp8" else 256


@pytest.mark.parametrize("codec", QCODECS)
@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("where", ["one", "three", "limit", "limit+1", "limit+3"])
def test_single_pass_forms_around_the_tile_limit(L, codec, N, where):
    lim = tile_form_limit(codec)
    tiles = {"one": 1, "three": 3, "limit": lim, "limit+1": lim + 1, "limit+3": lim + 3}[where]
    n = tiles * 2048
    xs = [adversarial_bf16(n, 7100 + 10 * N + r) if r % 2 == 0 else random_bf16(n, 7200 + r) for r in range(N)]
    outs, ws = run_allreduce(L, xs, codec, "auto")
    ref, used = O.allreduce(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(o, ref[0]), (codec, N, tiles)
    wb = L.lpar_wire_bytes(codec, n)
    host = ws.host()
    wires = [O.quantize(x, codec) for x in xs]
    for r in range(N):
        assert np.array_equal(host[r * wb:(r + 1) * wb], wires[r])
    assert np.array_equal(host[N * wb:(N + 1) * wb], O.reduce(wires, 0, tiles, codec))


# Seeded random cases over the whole argument space: codec, N in 1..8, 1..40
# tiles, every schedule (one-shot against its own oracle), a threshold either
# side of the message, in place or not; adversarial or random inputs per rank.
N_RANDOM_CASES = 48


@pytest.mark.parametrize("case", range(N_RANDOM_CASES))
def test_allreduce_random_cases(L, case):
    rng = np.random.default_rng(9000 + case)
    codec = CODECS[rng.integers(len(CODECS))]
    N = int(rng.integers(1, 9))
    tiles = int(rng.integers(1, 41))
    n = tiles * 2048
    schedule = ["auto", "fused", "three_stage", "single_pass", "one_shot"][rng.integers(5)]
    thr = [0, 2 * n, 2 * n + 2][rng.integers(3)]
    inplace = bool(rng.integers(2))
    xs = [adversarial_bf16(n, int(rng.integers(1 << 30))) if rng.integers(2)
          else random_bf16(n, int(rng.integers(1 << 30)), float(2.0 ** rng.integers(-8, 9))) for _ in range(N)]
    outs, _ = run_allreduce(L, xs, codec, schedule, thr, inplace)
    if schedule == "one_shot":
        ref, used = O.allreduce_oneshot(xs, codec, thr)
    else:
        ref, used = O.allreduce(xs, codec, thr)
    assert used == L.lpar_effective_codec(n, codec, thr)
    for o in outs:
        assert np.array_equal(o, ref[0]), (codec, N, tiles, schedule, thr, inplace)


# The same over 257..700 tiles per rank, where the persistent forms run (above
# the tile form's limit), with ragged last chunks and every schedule.
@pytest.mark.parametrize("case", range(16))
def test_allreduce_random_cases_persistent(L, case):
    rng = np.random.default_rng(9500 + case)
    codec = CODECS[rng.integers(len(CODECS))]
    N = int(rng.integers(1, 9))
    tiles = int(rng.integers(257, 701))
    n = tiles * 2048
    schedule = ["auto", "fused", "three_stage", "single_pass", "one_shot"][rng.integers(5)]
    inplace = bool(rng.integers(2))
    xs = [adversarial_bf16(n, int(rng.integers(1 << 30))) if rng.integers(2)
          else random_bf16(n, int(rng.integers(1 << 30)), float(2.0 ** rng.integers(-8, 9))) for _ in range(N)]
    outs, _ = run_allreduce(L, xs, codec, schedule, 0, inplace)
    ref, used = (O.allreduce_oneshot if schedule == "one_shot" else O.allreduce)(xs, codec)
    assert used == codec
    for o in outs:
        assert np.array_equal(o, ref[0]), (codec, N, tiles, schedule, inplace)


@pytest.mark.parametrize("codec", CODECS)
def test_allreduce_in_place(L, codec):
    n = 2048 * 6
    xs = [random_bf16(n, 700 + r, 2.0) for r in range(3)]
    outs, _ = run_allreduce(L, xs, codec, inplace=True)
    ref, _ = O.allreduce(xs, codec)
    for o in outs:
        assert np.array_equal(o, ref[0])


def test_threshold_sends_small_messages_to_bf16(L):
    w = W.WORKLOADS["decode_int3"]
    thr = w.min_quant_bytes
    for n, expect in ((w.n, "int3"), (w.n - 2048, "bf16")):
        xs = [t.view(torch.int16).numpy().view(np.uint16) for t in W.make_inputs(w, "cpu", n=n)]
        outs, _ = run_allreduce(L, xs, "int3", min_quant_bytes=thr)
        ref, used = O.allreduce(xs, "int3", min_quant_bytes=thr)
        assert used == expect
        assert np.array_equal(outs[0], ref[0]) and np.array_equal(outs[1], ref[0])


def test_empty_message_is_a_no_op(L):
    ws = Guarded(16)
    L.lpar_allreduce([ws.ptr()], 0, "int4", [ws.ptr()], ws.ptr(), 16)
    L.lpar_quantize(ws.ptr(), 0, "int3", ws.ptr())
    L.lpar_decode(ws.ptr(), 0, "fp8", ws.ptr())
    L.lpar_reduce([ws.ptr()], 0, 0, "int4", ws.ptr())
    torch.cuda.synchronize()
    assert torch.all(ws.buf == CANARY)


# ---------------------------------------------------------------------------
# The named workloads
# ---------------------------------------------------------------------------
def workload_bits(w, n=None):
    return [t.view(torch.int16).numpy().view(np.uint16) for t in W.make_inputs(w, "cpu", n=n)]


@pytest.mark.parametrize("name", ["small_int4", "decode_int3"])
def test_workload_full_oracle(L, name):
    w = W.WORKLOADS[name]
    xs = workload_bits(w)
    for codec in w.codecs:
        for schedule in ("fused", "three_stage", "single_pass"):
            outs, _ = run_allreduce(L, xs, codec, schedule, min_quant_bytes=w.min_quant_bytes)
            ref, used = O.allreduce(xs, codec, min_quant_bytes=w.min_quant_bytes)
            assert used == codec
            for o in outs:
                assert np.array_equal(o, ref[0])


def test_workload_prefill_fp8_full_oracle_and_error_report(L):
    w = W.WORKLOADS["prefill_fp8"]
    xs = workload_bits(w)
    exact = np.zeros(w.n, np.float64)
    for x in xs:
        exact += O.bf16_bits_to_f32(x).astype(np.float64)
    errs = {}
    for codec in w.codecs:                               # FP8, then the uncompressed BF16 sum
        outs, _ = run_allreduce(L, xs, codec)
        ref, _ = O.allreduce(xs, codec)
        for o in outs:
            assert np.array_equal(o, ref[0])
        e = O.bf16_bits_to_f32(outs[0]).astype(np.float64) - exact
        errs[codec] = (float(np.max(np.abs(e))), float(np.sqrt(np.mean(e * e))))
    print("prefill_fp8 error vs exact sum (max, rms):", errs)
    assert errs["bf16"][1] <= errs["fp8"][1]


@pytest.mark.parametrize("name", ["large_int3_int4", "large_mxfp4"])
def test_workload_large_sampled_tiles(L, name):
    """1 GiB per rank (INT3 then INT4, or MXFP4) in the launch configuration the
    bench times; compared on 1024 seeded random tiles plus the first and the
    last (tiles are independent, so a tile's result depends only on that tile
    of every rank)."""
    w = W.WORKLOADS[name]
    xs = W.make_inputs(w, "cuda")
    T = w.n // 2048
    rng = np.random.default_rng(4)
    tiles = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 1024, replace=False)]))
    idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
    sample_in = [x[idx].view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
    for codec in w.codecs:
        outs = [torch.empty_like(x) for x in xs]
        ws = torch.empty(L.lpar_workspace_bytes(w.N, w.n, codec), dtype=torch.uint8, device="cuda")
        ref, _ = O.allreduce(sample_in, codec)
        for schedule in ("fused", "single_pass"):
            L.lpar_allreduce(xs, w.n, codec, outs, ws, ws.numel(), schedule=schedule)
            torch.cuda.synchronize()
            for o in outs:
                got = o[idx].view(torch.int16).cpu().numpy().view(np.uint16)
                assert np.array_equal(got, ref[0]), (codec, schedule)
        del outs, ws
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# The single-pass kernel's CTA-wide form with bulk output copies (from 128 MiB
# of input, N x 2n; INT3 from 512 MiB and N >= 3) with odd rank counts and a
# ragged last chunk (T % 4 == 3); INT3 with N = 1 runs the warp-local form at
# every size.  Student-t inputs drawn on the GPU, with adversarial tiles
# planted at the sampled positions; sampled tiles are compared bit for bit.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "mxfp4"])
@pytest.mark.parametrize("N", [1, 3, 5])
def test_bulk_output_path_ragged_tail(L, codec, N):
    T = -(-((512 if codec == "int3" else 128) << 20) // (N * 4096))
    T += (3 - T % 4) % 4                             # T % 4 == 3: the last chunk holds three tiles
    assert N * T * 4096 >= (128 << 20) and T % 4 == 3
    n = T * 2048
    g = torch.Generator(device="cuda")
    xs = []
    for r in range(N):
        g.manual_seed(77 * 1009 + r)
        z = torch.randn(n, generator=g, device="cuda")
        c = sum(torch.randn(n, generator=g, device="cuda") ** 2 for _ in range(3))
        xs.append((z / torch.sqrt(c / 3)).to(torch.bfloat16))
    rng = np.random.default_rng(600 + N)
    tiles = np.unique(np.concatenate([np.arange(4), np.arange(T - 7, T), rng.choice(T, 48, replace=False)]))
    idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
    for r in range(N):                               # adversarial blocks at the sampled tiles
        adv = adversarial_bf16(len(tiles) * 2048, 6100 + 10 * N + r)
        xs[r][idx] = torch.from_numpy(adv.view(np.int16)).cuda().view(torch.bfloat16)
    sample_in = [x[idx].view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
    ref, _ = O.allreduce(sample_in, codec)
    outs = [torch.empty_like(x) for x in xs]
    ws = torch.empty(L.lpar_workspace_bytes(N, n, codec), dtype=torch.uint8, device="cuda")
    L.lpar_allreduce(xs, n, codec, outs, ws, ws.numel(), schedule="single_pass")
    torch.cuda.synchronize()
    for o in outs:
        assert np.array_equal(o[idx].view(torch.int16).cpu().numpy().view(np.uint16), ref[0]), (codec, N)
    del xs, outs, ws
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# The sweep: 128 KiB ... 1 GiB per rank, N in {2, 4, 8}, every codec, Student-t
# (nu = 3).  Each point runs at full size on the GPU.  Up to 64 MiB per rank the
# whole message is compared with the oracle (run over tile ranges on every host
# core); above, the first and last tile plus 1024 seeded random tiles (a tile's
# result depends only on that tile of every rank).  At every point the stage-1
# wires and the gathered wire (codes and scales) are compared byte for byte at
# the first and last tile and 1024 random ones (every tile of smaller messages).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N", list(W.SWEEP_RANKS))
def test_sweep_sampled_tiles(L, N):
    from oracle import parallel as OP
    rng = np.random.default_rng(5000 + N)
    for mb in W.SWEEP_SIZES_BYTES:
        w = W.sweep_workload(N, mb, "bf16")
        xs = W.make_inputs(w, "cuda")
        T = w.n // 2048
        full = mb <= (64 << 20)
        if full:
            host_in = [x.view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
            refs = OP.allreduce(host_in, list(W.SWEEP_CODECS))
            idx = None
        else:
            tiles = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 1024, replace=False)]))
            idx = torch.from_numpy((tiles[:, None] * 2048 + np.arange(2048)[None, :]).reshape(-1)).cuda()
            sample_in = [x[idx].view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
            refs = OP.allreduce(sample_in, list(W.SWEEP_CODECS))
        outs = [torch.empty_like(x) for x in xs]
        ws = torch.empty(max(L.lpar_workspace_bytes(N, w.n, c) for c in W.SWEEP_CODECS), dtype=torch.uint8,
                         device="cuda")
        # the stage-1 wires and the gathered wire (codes and scales) at the checked tiles: every
        # tile up to 1026 tiles, else the sampled ones
        wt = np.arange(T) if T <= 1026 else (
            tiles if not full else np.unique(np.concatenate([[0, T - 1], rng.choice(T, 1024, replace=False)])))
        if full:
            wsample = [h.reshape(T, 2048)[wt].reshape(-1) for h in host_in]
        else:
            pos = np.searchsorted(tiles, wt)
            wsample = [h.reshape(-1, 2048)[pos].reshape(-1) for h in sample_in]
        for codec in W.SWEEP_CODECS:
            if codec != "bf16":
                tb = L.lpar_tile_bytes(codec)
                wires = [O.quantize(x, codec) for x in wsample]
                gathered = O.reduce(wires, 0, len(wt), codec)
                byte_idx = torch.from_numpy((wt[:, None] * tb + np.arange(tb)[None, :]).reshape(-1)).cuda()
            for schedule in ("fused", "single_pass"):
                L.lpar_allreduce(xs, w.n, codec, outs, ws, ws.numel(), schedule=schedule)
                torch.cuda.synchronize()
                for o in outs:
                    g = o if idx is None else o[idx]
                    assert np.array_equal(g.view(torch.int16).cpu().numpy().view(np.uint16), refs[codec]), \
                        (N, mb, codec, schedule)
                if codec != "bf16":
                    wb = T * tb
                    for r in range(N + 1):                       # rank r's wire, then the gathered wire
                        got = ws[r * wb + byte_idx].cpu().numpy()
                        assert np.array_equal(got, wires[r] if r < N else gathered), (N, mb, codec, schedule, r)
        del xs, outs, ws
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Streams and graphs: the library never synchronises and keeps no per-call
# state, so calls on two streams at once, and calls captured in a CUDA graph
# and replayed on new inputs, give the oracle's results.
# ---------------------------------------------------------------------------
def test_two_streams_at_once(L):
    n = 2048 * 64
    jobs = []
    for k, codec in enumerate(("int3", "mxfp4")):
        xs = [adversarial_bf16(n, 1200 + 10 * k + r) for r in range(3)]
        dx = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs]
        outs = [torch.empty_like(d) for d in dx]
        ws = torch.empty(L.lpar_workspace_bytes(3, n, codec), dtype=torch.uint8, device="cuda")
        jobs.append((codec, xs, dx, outs, ws, torch.cuda.Stream()))
    torch.cuda.synchronize()
    for codec, xs, dx, outs, ws, s in jobs:
        for _ in range(3):                               # several calls in flight on each stream
            L.lpar_allreduce(dx, n, codec, outs, ws, ws.numel(), stream=s)
    torch.cuda.synchronize()
    for codec, xs, dx, outs, ws, s in jobs:
        ref, _ = O.allreduce(xs, codec)
        for o in outs:
            assert np.array_equal(o.cpu().numpy().view(np.uint16), ref[0])


@pytest.mark.parametrize("codec,schedule", [("int4", "auto"), ("fp8", "fused"), ("int3", "three_stage"),
                                            ("mxfp4", "one_shot")])
def test_captured_in_a_cuda_graph(L, codec, schedule):
    n, N = 2048 * 16, 2
    dx = [torch.empty(n, dtype=torch.int16, device="cuda") for _ in range(N)]
    outs = [torch.empty_like(d) for d in dx]
    ws = torch.empty(L.lpar_workspace_bytes(N, n, codec), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):                           # a first call outside capture fills the host caches
        L.lpar_allreduce(dx, n, codec, outs, ws, ws.numel(), schedule=schedule, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.lpar_allreduce(dx, n, codec, outs, ws, ws.numel(), schedule=schedule, stream=s)
    for k in range(2):                                   # replay on new inputs
        xs = [adversarial_bf16(n, 1300 + 10 * k + r) for r in range(N)]
        for d, x in zip(dx, xs):
            d.copy_(torch.from_numpy(x.view(np.int16)))
        g.replay()
        torch.cuda.synchronize()
        ref = (O.allreduce_oneshot if schedule == "one_shot" else O.allreduce)(xs, codec)[0]
        for o in outs:
            assert np.array_equal(o.cpu().numpy().view(np.uint16), ref[0])
