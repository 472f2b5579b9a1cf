"""The C ABI driven from plain C, with no Python in the loop (CPU only).

``tests/c_abi_trace.c`` is compiled with gcc against ``include/pagedkv.h``
and linked with ``libpagedkv.so``; it replays random allocator traces (adds,
one-token appends, prompt appends, forks, frees, running the pool dry, and
checkpoint/resume through ``pa_seqs_snapshot`` / ``pa_seqs_restore``) through
``pa_seqs_*`` / ``pa_alloc_*``.  Every result it prints, and the final
reference counts, free pool and block tables, must equal what the oracle
allocator gives for the same trace.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import allocator as AL
from paged_kv_cache_364_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def trace_exe(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    _lib.load()                                   # builds the library when it is missing
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path_factory.mktemp("c_abi") / "c_abi_trace")
    r = subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c_abi_trace.c"),
                        "-I", os.path.join(ROOT, "include"), "-L", libdir, "-lpagedkv", f"-Wl,-rpath,{libdir}",
                        "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def oracle_trace(seed, n_ops=400):
    """A random trace, the oracle allocator's answer to every operation, and
    its final state, in the C program's text format."""
    rng = np.random.default_rng(seed)
    nb, B = int(rng.integers(8, 64)), int(rng.choice([1, 4, 16]))
    order = rng.permutation(nb)
    pool = AL.BlockPool(nb, order)
    seqs = AL.SequenceTables(pool, B)
    ops = [f"O {nb} " + " ".join(str(int(b)) for b in order)]
    want = []
    live = []
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.1 or not live:
            sid = seqs.add()
            live.append(sid)
            ops.append("A")
            want.append(f"A {sid}")
        elif r < 0.6:
            sid = int(rng.choice(live))
            ops.append(f"P {sid}")
            try:
                slot, pair = seqs.append(sid)
                want.append(f"P {slot} {pair[0]} {pair[1]}" if pair is not None else f"P {slot} -1 -1")
            except AL.OutOfBlocks:
                want.append("P OOM")
        elif r < 0.7:
            sid, k = int(rng.choice(live)), int(rng.integers(1, 3 * B + 2))
            ops.append(f"N {sid} {k}")
            placed, copies = [], 0
            try:
                for _ in range(k):
                    slot, pair = seqs.append(sid)
                    placed.append(slot)
                    copies += pair is not None
                want.append(f"N {placed[0]} {placed[-1]} {copies}")
            except AL.OutOfBlocks:              # the tokens placed before the failing one stay
                want.append("N OOM")
        elif r < 0.73:
            # checkpoint and resume; the snapshot holds a 7-word header, the
            # free pool, the counts, and 3 words plus the blocks per table
            ops.append("R")
            words = 7 + len(pool.free) + nb + sum(3 + len(t) for t in seqs.tables.values())
            want.append(f"R {4 * words}")
        elif r < 0.85:
            sid = int(rng.choice(live))
            child = seqs.fork(sid)
            live.append(child)
            ops.append(f"F {sid}")
            want.append(f"F {child}")
        else:
            sid = live.pop(int(rng.integers(len(live))))
            seqs.free(sid)
            ops.append(f"X {sid}")
            want.append("X")
    want.append(f"RC {nb} " + " ".join(str(c) for c in pool.refcount))
    want.append(f"FREE {len(pool.free)}" + "".join(f" {b}" for b in pool.free))
    for sid in sorted(seqs.tables):
        table = seqs.tables[sid]
        want.append(f"T {sid} {seqs.lens[sid]} {len(table)}" + "".join(f" {b}" for b in table))
    return nb, B, "\n".join(ops) + "\n", want


@pytest.mark.parametrize("seed", range(6))
def test_c_program_matches_the_oracle_allocator(trace_exe, seed):
    nb, B, trace, want = oracle_trace(2000 + seed)
    r = subprocess.run([trace_exe, str(nb), str(B)], input=trace, capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    got = r.stdout.strip().splitlines()
    assert len(got) == len(want)
    for i, (g, w) in enumerate(zip(got, want)):
        assert g == w, f"line {i}: {g!r} != {w!r}"
    assert any(line.endswith("OOM") for line in want)                   # the pool ran dry somewhere


def test_c_program_rejects_a_trace_without_the_pool_order(trace_exe):
    r = subprocess.run([trace_exe, "8", "4"], input="A\n", capture_output=True, text=True, timeout=60)
    assert r.returncode == 1 and "free order" in r.stderr
