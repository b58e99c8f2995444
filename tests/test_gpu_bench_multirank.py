"""bench.py --gpus 2 end to end on the one GPU (needs a B200): torchrun starts two
ranks, both on cuda:0, with the gloo backend (the wire bytes move through host
copies; no kernel waits on another process), and rank 0 prints the bench line of
the real cross-rank all-reduce.  The line must follow the bench contract: the
aggregate over both ranks, the NVLink roofline, the e2e block and no CPU
baseline."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_bench_two_ranks_one_gpu():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--steps", "3", "--warmup", "3", "--workload", "small_int4", "--backend", "gloo", "--chunks", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["steps"] == 3 and d["scaling"] == "weak"
    assert d["config"]["ranks"] == 2 and d["config"]["workload"] == "small_int4"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # whole-job throughput: both ranks' messages over the slowest rank's time
    assert d["value"] == pytest.approx(2 * 65536 * 2 / (d["ms_per_step"] * 1e-3) / 1e9, rel=1e-6)
    assert d["roofline"]["bound"] == "nvlink" and d["roofline"]["achieved"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 65536 * 2 and d["e2e"]["value"] > 0
    assert d["cpu_baseline"] is None and d["gpu_launches"] > 0
