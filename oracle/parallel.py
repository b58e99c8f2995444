"""The oracle's all-reduce over tile ranges on all host cores.  TEST
INFRASTRUCTURE ONLY (the CPU-baseline legs of ``bench.py`` time it; the GPU
parity tests use `allreduce` to check whole messages against it).

Every tile of the collective depends only on the same tile of every rank, so
the oracle's all-reduce of a tile range is exactly its share of the whole call.
``run`` splits the tiles into one contiguous range per worker, hands the
inputs over in a memory-mapped file (in /dev/shm where there is one; each
worker copies its range out before the timed span), starts all workers
together and reports the span from the first start to the last end.
The oracle itself is unchanged: each worker calls it single-threaded on its
range.  Workers are fresh interpreters (``python -c``) that import only numpy
and the oracle: no CUDA state and no caller module is inherited.
"""
import os
import selectors
import subprocess
import sys
import tempfile
import time

import numpy as np

from . import oracle as O

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _worker_main(argv=None):
    """Worker: copy its tile range out of the mapped file, run the warm-up,
    print `ready`, wait for a line on stdin, run, print `done <start> <end>`
    (perf_counter seconds)."""
    path, N, n, dtype, t0, t1, codecs, f32, warmup, repeat = (argv or sys.argv[1:])
    N, n, t0, t1, warmup, repeat = int(N), int(n), int(t0), int(t1), int(warmup), int(repeat)
    f32 = f32 == "1"
    codecs = codecs.split(",")
    arr = np.memmap(path, dtype=np.dtype(dtype), mode="r", shape=(N, n))
    xs = [np.array(arr[r, t0 * O.TILE_ELEMS:t1 * O.TILE_ELEMS]) for r in range(N)]   # this worker's range
    del arr
    fn = O.allreduce_f32 if f32 else O.allreduce
    for _ in range(warmup):
        for c in codecs:
            fn(xs, c, 0)
    print("ready", flush=True)
    sys.stdin.readline()
    a = time.perf_counter()
    for _ in range(repeat):
        for c in codecs:
            fn(xs, c, 0)
    b = time.perf_counter()
    print("done %.9f %.9f" % (a, b), flush=True)


def _compute_main(argv=None):
    """Worker of `allreduce`: the oracle's all-reduce of its tile range with
    each codec in turn, written into the output file at that range (rank 0's
    output: every rank receives the same values); prints `done`."""
    in_path, out_path, N, n, t0, t1, codecs = (argv or sys.argv[1:])
    N, n, t0, t1 = int(N), int(n), int(t0), int(t1)
    codecs = codecs.split(",")
    arr = np.memmap(in_path, dtype=np.uint16, mode="r", shape=(N, n))
    xs = [np.array(arr[r, t0 * O.TILE_ELEMS:t1 * O.TILE_ELEMS]) for r in range(N)]
    del arr
    res = np.memmap(out_path, dtype=np.uint16, mode="r+", shape=(len(codecs), n))
    for k, c in enumerate(codecs):
        outs, _ = O.allreduce(xs, c, 0)
        res[k, t0 * O.TILE_ELEMS:t1 * O.TILE_ELEMS] = outs[0]
    res.flush()
    del res
    print("done 0 0", flush=True)


def allreduce(xs, codecs, workers=None, timeout=1800.0):
    """The oracle's all-reduce of the N host arrays `xs` (BF16 bits as uint16,
    whole tiles) for every codec of `codecs` (each the codec the message runs
    with: no threshold), over tile ranges on every host core.  Returns
    {codec: the result every rank receives}."""
    N, n = len(xs), xs[0].size
    T = n // O.TILE_ELEMS
    P = max(1, min(workers or host_cores(), T))
    O.lib()
    tmpdir = "/dev/shm" if os.path.isdir("/dev/shm") else None
    paths = []
    procs = []
    try:
        for suffix in (".in", ".out"):
            fd, path = tempfile.mkstemp(prefix="lpar_oracle_", suffix=suffix, dir=tmpdir)
            os.close(fd)
            paths.append(path)
        arr = np.memmap(paths[0], dtype=np.uint16, mode="w+", shape=(N, n))
        for r, x in enumerate(xs):
            arr[r] = np.asarray(x, dtype=np.uint16).reshape(-1)
        arr.flush()
        del arr
        res = np.memmap(paths[1], dtype=np.uint16, mode="w+", shape=(len(codecs), n))
        res.flush()
        del res
        env = dict(os.environ, PYTHONPATH=_ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
        for k in range(P):
            t0, t1 = k * T // P, (k + 1) * T // P
            args = [paths[0], paths[1], N, n, t0, t1, ",".join(codecs)]
            procs.append(subprocess.Popen(
                [sys.executable, "-c", "from oracle.parallel import _compute_main; _compute_main()"] + [str(a) for a in args],
                stdin=subprocess.DEVNULL, stdout=subprocess.PIPE, text=True, env=env, cwd=_ROOT))
        _read_lines(procs, "done", time.monotonic() + timeout)
        for p in procs:
            p.wait(timeout=60)
        res = np.array(np.memmap(paths[1], dtype=np.uint16, mode="r", shape=(len(codecs), n)))
        return {c: res[k] for k, c in enumerate(codecs)}
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
                p.wait()
        for path in paths:
            os.unlink(path)


def _read_lines(procs, want, deadline):
    """One line from each worker's stdout, starting with `want`."""
    sel = selectors.DefaultSelector()
    for i, p in enumerate(procs):
        sel.register(p.stdout, selectors.EVENT_READ, i)
    got = {}
    try:
        while len(got) < len(procs):
            left = deadline - time.monotonic()
            if left <= 0:
                raise RuntimeError("oracle workers did not answer in time")
            for key, _ in sel.select(timeout=min(left, 5.0)):
                line = key.fileobj.readline()
                if not line.startswith(want):
                    raise RuntimeError("oracle worker %d failed (exit %s)" % (key.data, procs[key.data].poll()))
                got[key.data] = line.split()[1:]
                sel.unregister(key.fileobj)
    finally:
        sel.close()
    return [got[i] for i in range(len(procs))]


def run(xs, codecs, f32=False, workers=None, warmup=0, repeat=1, timeout=1800.0):
    """All-reduce of the N host arrays `xs` (BF16 bits as uint16, or binary32;
    whole tiles) with each codec of `codecs` in turn, `repeat` times, split over
    `workers` processes (default: every host core, at most one per tile).  Each
    codec must be the one the whole message runs with: the slices are called
    with no threshold.  Returns (seconds, workers used)."""
    N, n = len(xs), xs[0].size
    T = n // O.TILE_ELEMS
    P = max(1, min(workers or host_cores(), T))
    dtype = np.dtype(np.float32 if f32 else np.uint16)
    O.lib()                             # build the oracle once, before the workers load it
    tmpdir = "/dev/shm" if os.path.isdir("/dev/shm") else None
    fd, path = tempfile.mkstemp(prefix="lpar_oracle_", suffix=".bin", dir=tmpdir)
    os.close(fd)
    procs = []
    try:
        arr = np.memmap(path, dtype=dtype, mode="w+", shape=(N, n))
        for r, x in enumerate(xs):
            arr[r] = np.asarray(x, dtype=dtype).reshape(-1)
        arr.flush()
        del arr
        env = dict(os.environ, PYTHONPATH=_ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
        for k in range(P):
            t0, t1 = k * T // P, (k + 1) * T // P
            args = [path, N, n, dtype.name, t0, t1, ",".join(codecs), int(f32), warmup, repeat]
            procs.append(subprocess.Popen(
                [sys.executable, "-c", "from oracle.parallel import _worker_main; _worker_main()"] + [str(a) for a in args],
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True, env=env, cwd=_ROOT))
        deadline = time.monotonic() + timeout
        _read_lines(procs, "ready", deadline)
        for p in procs:
            p.stdin.write("go\n")
            p.stdin.flush()
        spans = [(float(a), float(b)) for a, b in _read_lines(procs, "done", deadline)]
        for p in procs:
            p.wait(timeout=max(1.0, deadline - time.monotonic()))
        return max(b for _, b in spans) - min(a for a, _ in spans), P
    finally:
        for p in procs:                 # only the processes started here
            if p.poll() is None:
                p.kill()
                p.wait()
        os.unlink(path)
