"""The all-cores CPU baseline: the oracle over tile ranges (CPU only).

The parallel runner is valid only because a tile's result depends on nothing
but the same tile of every rank; that premise is checked here against whole
calls of the oracle, for every codec and operation the baseline runs, then the
runner itself is exercised (worker processes, hand-over, timing) and the
reference arm of bench.py is run end to end.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from oracle import oracle as O
from oracle import parallel as OP

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TILE = O.TILE_ELEMS


def bf16_inputs(N, T, seed):
    rng = np.random.default_rng(seed)
    return [(rng.standard_t(3, T * TILE).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
            for _ in range(N)]


@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "mxfp4", "bf16"])
@pytest.mark.parametrize("N", [2, 3])
def test_tile_range_equals_slice_of_whole_call(codec, N):
    T = 7
    xs = bf16_inputs(N, T, 40 + N)
    whole, _ = O.allreduce(xs, codec)
    for t0, t1 in [(0, 3), (3, 4), (4, 7)]:
        part, _ = O.allreduce([x[t0 * TILE:t1 * TILE] for x in xs], codec)
        for p, w in zip(part, whole):
            assert np.array_equal(p, w[t0 * TILE:t1 * TILE])


@pytest.mark.parametrize("codec", ["fp8", "bf16"])
def test_tile_range_equals_slice_binary32(codec):
    rng = np.random.default_rng(5)
    xs = [rng.standard_normal(5 * TILE).astype(np.float32) for _ in range(3)]
    whole, _ = O.allreduce_f32(xs, codec)
    part, _ = O.allreduce_f32([x[2 * TILE:5 * TILE] for x in xs], codec)
    for p, w in zip(part, whole):
        assert np.array_equal(p.view(np.uint32), w[2 * TILE:5 * TILE].view(np.uint32))


def test_runner_splits_over_workers():
    xs = bf16_inputs(2, 6, 1)
    dt, used = OP.run(xs, ["int3", "int4"], workers=3)
    assert used == 3 and dt > 0
    dt, used = OP.run(xs, ["int3"], workers=64, warmup=1, repeat=2)
    assert used == 6 and dt > 0                   # at most one worker per tile
    xf = [np.random.default_rng(2).standard_normal(2 * TILE).astype(np.float32) for _ in range(2)]
    dt, used = OP.run(xf, ["fp8"], f32=True, workers=2)
    assert used == 2 and dt > 0


def test_whole_message_over_workers_equals_one_call():
    xs = bf16_inputs(3, 11, 21)
    codecs = ["int4", "int3", "fp8", "mxfp4", "bf16"]
    got = OP.allreduce(xs, codecs, workers=4)
    for c in codecs:
        ref, _ = O.allreduce(xs, c)
        assert np.array_equal(got[c], ref[0]), c


def test_runner_reports_a_failing_worker():
    xs = bf16_inputs(2, 2, 3)
    with pytest.raises(RuntimeError):
        OP.run(xs, ["no_such_codec"], workers=2, timeout=120)


def test_reference_arm_prints_one_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "decode_int3",
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0
