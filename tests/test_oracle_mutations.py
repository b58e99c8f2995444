"""Every planted mistake in the oracle fails at least one committed pin (CPU only).

For each entry of tests/oracle_mutations.py a copy of oracle/lpar_oracle.c is
edited, compiled with the oracle's own flags, and the pin files named for its
group are run against it in a child pytest (the oracle loader takes the
library path from LPAR_ORACLE_LIB).  A mutation counts as caught when that run
fails.  The copies are built and run in parallel, one child per host core.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle import build_oracle
from tests import oracle_mutations as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lpar_oracle.c")
HDR = os.path.join(ROOT, "oracle", "lpar_oracle.h")

CASES = [(name, edits, files) for group, files in M.GROUPS for name, edits in group]


def _mutate(src, edits):
    for old, new in edits:
        if old not in src:
            raise AssertionError("mutation text no longer in the oracle source: %r" % old[:60])
        src = src.replace(old, new, 1)
    return src


def _run_one(workdir, idx, name, edits, files):
    d = os.path.join(workdir, "m%03d" % idx)
    os.makedirs(d, exist_ok=True)
    with open(SRC) as f:
        src = _mutate(f.read(), edits)
    with open(os.path.join(d, "lpar_oracle.c"), "w") as f:
        f.write(src)
    with open(HDR) as f, open(os.path.join(d, "lpar_oracle.h"), "w") as g:
        g.write(f.read())
    lib = os.path.join(d, "liblpar_oracle.so")
    cc = subprocess.run(["gcc", *build_oracle.CFLAGS, os.path.join(d, "lpar_oracle.c"), "-o", lib, "-lm"],
                        capture_output=True, text=True)
    if cc.returncode != 0:
        return ("does not compile", cc.stderr[-400:])
    env = dict(os.environ, LPAR_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *[os.path.join(ROOT, "tests", f) for f in files]],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = [line for line in r.stdout.splitlines() if line.startswith("FAILED")]
    return ("caught" if r.returncode != 0 else "missed", failed[:1])


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    workdir = str(tmp_path_factory.mktemp("oracle_mutations"))
    jobs = max(1, min(len(CASES), os.cpu_count() or 1))
    with ThreadPoolExecutor(jobs) as pool:
        futs = {name: pool.submit(_run_one, workdir, i, name, edits, files)
                for i, (name, edits, files) in enumerate(CASES)}
        return {name: f.result() for name, f in futs.items()}


def test_names_are_unique():
    names = [c[0] for c in CASES]
    assert len(names) == len(set(names))


@pytest.mark.parametrize("name", [c[0] for c in CASES])
def test_mutation_is_caught(outcomes, name):
    verdict, detail = outcomes[name]
    assert verdict == "caught", "%s: %s %s" % (name, verdict, detail)
