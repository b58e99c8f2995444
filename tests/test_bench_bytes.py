"""bench.py's byte model on the host (no GPU): the algorithmic bytes behind every
roofline fraction, checked against the per-element model they come from (stage-1
wires written and read back, one gathered wire, N outputs), and the kernel labels
against the library's choice of form."""
import os
import random
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

C = bench.CODEC_C


def test_wire_bytes_per_element_are_the_tile_sizes():
    assert C["int4"] * 2048 == 1152 and C["int3"] * 2048 == 896
    assert C["fp8"] * 2048 == 2304 and C["mxfp4"] * 2048 == 1088 and C["bf16"] == 2


@pytest.mark.parametrize("codec", ["int4", "int3", "fp8", "mxfp4"])
def test_single_pass_bytes_follow_the_per_element_model(codec):
    # per N*n elements: 2 in + c wire out + c wire back in + c/N gathered wire + 2 out
    rng = random.Random(1)
    for _ in range(50):
        N = rng.randint(1, 8)
        n = 2048 * rng.randint(1, 1 << 18)
        c = C[codec]
        got = bench.algorithmic_bytes("k_allreduce_single<%s,N=%d>" % (codec, N), codec, N, n)
        assert got == pytest.approx(N * n * (4 + 2 * c + c / N))
        assert bench.algorithmic_bytes("k_allreduce_single_warp<%s,N=%d>" % (codec, N), codec, N, n) == got


def test_schedules_move_the_same_bytes_as_single_pass():
    N, n = 4, 2048 * 1000
    for codec in ("int4", "int3", "fp8", "mxfp4"):
        single = bench.algorithmic_bytes("k_allreduce_single<x>", codec, N, n)
        fused = sum(bench.algorithmic_bytes(k, codec, N, n) for k in bench.kernel_names(codec, "fused", N))
        three = sum(bench.algorithmic_bytes(k, codec, N, n) for k in bench.kernel_names(codec, "three_stage", N))
        assert fused == pytest.approx(single)
        assert three == pytest.approx(single + n * C[codec])  # K3 also reads the gathered wire


def test_binary32_bytes():
    N, n = 8, 2048 * 8192
    c = C["fp8"]
    assert bench.algorithmic_bytes("k_allreduce_single_f32<fp8,N=8>", "fp8", N, n) == \
        pytest.approx(N * n * (4 + c) + n * (N * c + c + 4 * N))
    assert bench.algorithmic_bytes("k_f32_reduce<N=8>", "bf16", N, n) == n * (8 * N + 4)


def test_bench_workload_bytes():
    """The per-launch algorithmic bytes of the default bench workload (N = 2 x 512 Mi)."""
    n = 512 * 1024 * 1024
    assert bench.algorithmic_bytes("k_allreduce_single_warp<int3,N=2>", "int3", 2, n) == 5469372416
    assert bench.algorithmic_bytes("k_allreduce_single<int4,N=2>", "int4", 2, n) == 5804916736
    assert bench.algorithmic_bytes("k_allreduce_single<mxfp4,N=2>", "mxfp4", 2, n) == 5721030656


def test_collective_bytes():
    N, m = 4, 2048 * 100
    c = C["int3"]
    assert bench.collective_bytes("reduce_scatter", "int3", N, m) == pytest.approx(N * m * (2 + c) + N * m * c + 2 * m)
    assert bench.collective_bytes("one_shot", "int3", N, m) == pytest.approx(N * m * (2 + 2 * c) + 2 * N * m)
    assert bench.collective_bytes("all_gather", "int3", N, m) == pytest.approx(N * m * (2 + c) + 2 * N * N * m)
    assert bench.collective_bytes("all_to_all", "int3", N, m) == pytest.approx(N * N * m * (2 + c) + 2 * N * N * m)
    assert bench.collective_bytes("all_gather", "bf16", N, m) == N * 2 * m + 2 * N * N * m
    # the peer-memory all-reduce in one GPU: inputs, mailboxes written and read, N gathered
    # copies written and read, outputs
    assert bench.collective_bytes("peer_allreduce", "int3", N, m) == pytest.approx(
        N * 2 * m + N * m * c + N * m * c + N * m * c + N * m * c + N * 2 * m)
    assert bench.collective_bytes("peer_allreduce", "bf16", N, m) == N * m * 12


def test_peer_bytes_sent():
    """Per rank: its wire tiles of the other shards, and its reduced shard to the N - 1 others."""
    T, tb = 10, 896
    n = T * 2048
    assert bench.peer_bytes_sent(3, n, "int3", 0) == (10 - 3) * tb + 2 * 3 * tb     # shard 0 = tiles [0, 3)
    assert bench.peer_bytes_sent(3, n, "int3", 2) == (10 - 4) * tb + 2 * 4 * tb     # shard 2 = tiles [6, 10)
    assert bench.peer_bytes_sent(1, n, "int4", 0) == 0


def test_single_pass_labels_follow_the_launcher_rule():
    mib = 1 << 20
    k = bench.single_pass_kernel
    assert k("int4", 8, 256 * 2048).startswith("k_allreduce_tile")              # 256 tiles per rank
    assert k("int4", 2, 257 * 2048).startswith("k_allreduce_single_warp")       # 257
    assert k("fp8", 4, 512 * 2048).startswith("k_allreduce_tile")               # FP8: up to 512 tiles
    assert k("fp8", 4, 513 * 2048).startswith("k_allreduce_single<")
    assert k("int3", 2, 512 * mib).startswith("k_allreduce_single_warp")        # INT3, N <= 2: always
    assert k("int3", 8, 16 * mib).startswith("k_allreduce_single_warp")         # 256 MiB < 512 MiB of input
    assert k("int3", 8, 64 * mib).startswith("k_allreduce_single<")             # 1 GiB of input
    assert k("int4", 2, 16 * mib).startswith("k_allreduce_single_warp")         # 64 MiB < 128 MiB
    assert k("int4", 2, 32 * mib).startswith("k_allreduce_single<")             # 128 MiB
    assert k("mxfp4", 4, 8 * mib).startswith("k_allreduce_single_warp")
    assert k("fp8", 2, 2048 * 2048).startswith("k_allreduce_single<")           # FP8 above the tile form: CTA-wide
    src = open(os.path.join(ROOT, "quantized_precision_all_b200", "csrc", "lpar_kernels.cu")).read()
    assert "kBulkMinBytes = (size_t)128 << 20" in src and "kInt3WarpMaxBytes = (size_t)512 << 20" in src
    tiles_src = open(os.path.join(ROOT, "quantized_precision_all_b200", "csrc", "lpar_tiles.cuh")).read()
    assert "return C == kFP8 ? 512 : 256;" in tiles_src
    assert bench.BULK_MIN_BYTES == 128 * mib and bench.INT3_WARP_MAX_BYTES == 512 * mib


def test_input_digests_name_the_exact_bytes():
    import hashlib
    import torch
    import workloads as W
    w = W.WORKLOADS["small_int4"]
    xs = W.make_inputs(w, "cpu")
    d = bench.input_digests(w, xs)
    for r, x in enumerate(xs):
        assert d[r]["seed"] == w.seed * 1009 + r
        assert d[r]["sha256"] == hashlib.sha256(x.view(torch.int16).numpy().tobytes()).hexdigest()
    assert d[0]["sha256"] != d[1]["sha256"]


def test_buffer_sets_span_four_l2_at_distinct_addresses():
    """The rotated buffer sets of back-to-back timing: at least 512 MiB in all (4x the
    126 MB L2), every set's inputs equal to the originals, no two buffers sharing
    bytes; a workload already larger than that gets one set (its own buffers)."""
    import torch
    N, n = 2, 2048 * 64                                    # 256 KiB of BF16 per rank
    xs = [torch.full((n,), float(r + 1), dtype=torch.bfloat16) for r in range(N)]
    sets = bench.BufferSets(xs, n, 4096, torch.device("cpu"), rotate=8 << 20)
    set_bytes = N * n * 2 + N * n * 2 + 4096
    assert sets.R == -(-(8 << 20) // set_bytes) and sets.R * set_bytes >= 8 << 20
    spans = []
    for i in range(sets.R):
        for r in range(N):
            assert torch.equal(sets.inputs[i][r], xs[r])
            t = sets.inputs[i][r]
            spans.append((t.data_ptr(), t.data_ptr() + t.numel() * 2))
            o = sets.outputs[i][r]
            spans.append((o.data_ptr(), o.data_ptr() + o.numel() * 2))
        spans.append((sets.ws[i].data_ptr(), sets.ws[i].data_ptr() + sets.ws_bytes))
    spans.sort()
    assert all(a1 <= b0 for (a0, a1), (b0, b1) in zip(spans, spans[1:]))
    assert bench.ROTATE_BYTES == 512 << 20
    big = bench.BufferSets(xs, n, 4096, torch.device("cpu"), rotate=1024)
    assert big.R == 1 and big.inputs[0][0] is xs[0]


def test_min_dram_bytes():
    """Inputs read once, the N stage-1 wires and the gathered wire written once, the N
    outputs written (the wires' read-back may come from L2); BF16 has no stage-1 wire."""
    n = 2048 * 10
    assert bench.min_dram_bytes("int4", 2, n) == 2 * 2 * n + 2 * 10 * 1152 + 10 * 1152 + 2 * 2 * n
    assert bench.min_dram_bytes("fp8", 8, n) == 8 * 2 * n + 8 * 10 * 2304 + 10 * 2304 + 8 * 2 * n
    assert bench.min_dram_bytes("bf16", 4, n) == 4 * 2 * n + 2 * n + 4 * 2 * n


def test_nvlink_bytes_sent():
    """Per rank and chunk: its wire minus its own shard (the all-to-all), then its
    padded shard to each of the other ranks (the all-gather)."""
    tb = 1152
    n = 2048 * 10
    # one chunk, 2 ranks: shards [0, 5), [5, 10)
    assert bench.nvlink_bytes_sent(2, n, "int4", 1, 0) == 10 * tb - 5 * tb + 1 * 5 * tb
    # 3 ranks: shards [0, 3), [3, 6), [6, 10); slots padded to 4 tiles
    assert bench.nvlink_bytes_sent(3, n, "int4", 1, 0) == 10 * tb - 3 * tb + 2 * 4 * tb
    assert bench.nvlink_bytes_sent(3, n, "int4", 1, 2) == 10 * tb - 4 * tb + 2 * 4 * tb
    # two chunks of 5 tiles, 2 ranks: shards [0, 2), [2, 5) in each, slots of 3 tiles
    assert bench.nvlink_bytes_sent(2, n, "int4", 2, 0) == 2 * (5 * tb - 2 * tb + 3 * tb)


def test_distributed_line_carries_the_contract_keys():
    """The multi-GPU JSON line: the contract's keys, the whole-job value, an NVLink roofline."""
    import argparse
    import workloads as W
    w = W.WORKLOADS["large_int3_int4"]
    args = argparse.Namespace(steps=10, warmup=3, schedule="auto", backend="nccl", chunks=4, exchange="peer")
    res = {"w": w, "ms": 50.0, "sent": 10 ** 9, "launches_per_step": 2, "clocks": {"sm_mhz": 1965.0},
           "e2e": None, "exchange": "peer"}
    line = bench.distributed_line(args, 4, res)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks", "e2e"):
        assert k in line, k
    assert line["n_gpus"] == 4 and line["scaling"] == "weak" and line["gpu_launches"] == 20
    assert line["value"] == pytest.approx(4 * w.message_bytes * len(w.codecs) * 10 / 50e-3 / 1e9)
    rf = line["roofline"]
    assert rf["bound"] == "nvlink" and rf["peak"] == bench.NVLINK_GBS
    assert rf["achieved"] == pytest.approx(10 ** 9 / 5e-3 / 1e9) and rf["frac"] == pytest.approx(rf["achieved"] / 770.0)
    assert line["config"]["exchange"] == "peer" and line["config"]["ranks"] == 4


def test_clock_summary_from_samples():
    """The clock record: median SM clock, the highest max clock, every throttle reason
    seen Active, malformed lines skipped; no samples gives an empty record."""
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.lines = ["1965, 1965, 812.4, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
                "1710, 1965, 999.8, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
                "1800, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
                "garbage line",
                "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    s = cs.summary()
    assert s == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    cs.lines = ["1500, 1965, 700, 0x8, Active, Not Active, Active, Not Active"]
    assert cs.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    cs.lines = []
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_emulation_line_carries_the_contract_keys():
    """The one-GPU JSON line: the contract's keys, the whole-job value, and the roofline of
    the dominant kernel from its live launch time and the committed ncu traffic."""
    import argparse
    import workloads as W
    w = W.WORKLOADS["large_int3_int4"]
    args = argparse.Namespace(steps=20, warmup=3, schedule="auto", eager=False)
    n = w.n
    kern = {}
    for k, ms in (("k_allreduce_single_warp<int3,N=2>", 0.86), ("k_allreduce_single<int4,N=2>", 0.88)):
        codec = "int3" if "int3" in k else "int4"
        alg = bench.algorithmic_bytes(k, codec, 2, n)
        kern[k] = {"ms_total": ms * 20, "launches": 20, "ms_per_launch": ms, "algorithmic_bytes": alg,
                   "min_dram_bytes": bench.min_dram_bytes(codec, 2, n), "achieved_gbs": alg / (ms * 1e-3) / 1e9}
    res = {"w": w, "ms": 1.74 * 20, "kern": kern, "clocks": {"sm_mhz": 1965.0, "reasons": []},
           "launches_per_step": 2, "e2e": {"value": 45.0}, "cpu": {"value": 0.6}, "accuracy": None, "sets": 1,
           "inputs": [{"rank": 0, "seed": 4036, "sha256": "x"}]}
    line = bench.emulation_line(args, res)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks", "e2e", "cpu_baseline"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["gpu_launches"] == 40
    assert line["value"] == pytest.approx(2 * w.message_bytes * 2 / 1.74e-3 / 1e9)
    rf = line["roofline"]
    assert rf["kernel"] == "k_allreduce_single<int4,N=2>" and rf["bound"] == "hbm"
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"])
    for k in ("achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf
    assert line["config"]["inputs"][0]["seed"] == 4036
