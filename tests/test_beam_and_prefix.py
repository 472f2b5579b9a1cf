"""Beam search and prefix sharing on the block allocator.

"Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention", Technical
Details, "Beam Search Optimization": beams that share history share physical
blocks; pruned beams decrement reference counts and blocks reaching zero
return to the free pool; a branching event needs at most one block copy per
new branch.  "49 vLLM / PagedAttention", "Questions worth asking": a long
common system prompt can be stored once and referenced by every request.

CPU tests drive random beam-search process trees through the C++ allocator and
the oracle allocator and require identical tables, counts and free pools; the
GPU test also writes and copies real K/V and checks caches and decode.
"""

import numpy as np
import pytest

import paged_kv_cache_364_b200 as pk
from oracle import allocator as OAL


def beam_trace(seed, width=4, steps=60, prompt=37, B=8, nb=400):
    """Yields (op, args) of a beam search: each step every beam appends one
    token, then beams are re-selected (parents with several children fork,
    parents with none are freed)."""
    rng = np.random.default_rng(seed)
    ops = [("add",), ("append_n", 0, prompt)]
    beams = [0]
    next_id = 1
    for _ in range(steps):
        ops.append(("append", list(beams)))
        # choose parents of the next width beams (with replacement, like top-k over candidates)
        parents = sorted(rng.choice(len(beams), size=width, replace=True).tolist())
        counts = np.bincount(parents, minlength=len(beams))
        new_beams = []
        for i, b in enumerate(beams):
            for c in range(counts[i]):
                if c == 0:
                    new_beams.append(b)
                else:
                    ops.append(("fork", b, next_id))
                    new_beams.append(next_id)
                    next_id += 1
        for i, b in enumerate(beams):
            if counts[i] == 0:
                ops.append(("free", b))
        beams = new_beams
    return ops, nb, B


def replay(ops, nb, B, lib):
    if lib:
        pool = pk.BlockPool(nb, np.random.default_rng(0).permutation(nb))
        seqs = pk.SequenceTables(pool, B)
    else:
        pool = OAL.BlockPool(nb, np.random.default_rng(0).permutation(nb))
        seqs = OAL.SequenceTables(pool, B)
    copies_per_event = []
    for op in ops:
        if op[0] == "add":
            seqs.add()
        elif op[0] == "append_n":
            if lib:
                seqs.append_n(op[1], op[2])
            else:
                for _ in range(op[2]):
                    seqs.append(op[1])
        elif op[0] == "append":
            if lib:
                _, pairs = seqs.append(op[1])
            else:
                _, pairs = seqs.append_many(op[1])
            copies_per_event.append(len(pairs))
        elif op[0] == "fork":
            assert seqs.fork(op[1]) == op[2]
        elif op[0] == "free":
            seqs.free(op[1])
    if lib:
        live = seqs.live()
        state = (pool.refcounts(), pool.free_list(), {s: seqs.table(s) for s in live})
    else:
        live = sorted(seqs.tables)
        state = (list(pool.refcount), list(pool.free), {s: seqs.table(s) for s in live})
    return state, copies_per_event


@pytest.mark.parametrize("seed", range(6))
def test_beam_search_trees_match_the_oracle(seed):
    ops, nb, B = beam_trace(seed)
    got, got_copies = replay(ops, nb, B, lib=True)
    want, want_copies = replay(ops, nb, B, lib=False)
    assert got == want and got_copies == want_copies


@pytest.mark.parametrize("seed", range(3))
def test_one_block_copy_per_new_branch(seed):
    """Copies made by a step never exceed the forks made at the previous
    branching event, and blocks of pruned beams go back to the pool."""
    ops, nb, B = beam_trace(seed, width=5, steps=40)
    forks_before = []
    n_forks = 0
    for op in ops:
        if op[0] == "fork":
            n_forks += 1
        elif op[0] == "append":
            forks_before.append(n_forks)
            n_forks = 0
    (rc, free, tables), copies = replay(ops, nb, B, lib=True)
    for c, f in zip(copies, forks_before):
        assert c <= f
    live_refs = sum(len(t) for t in tables.values())
    assert sum(rc) == live_refs
    assert len(free) == nb - sum(1 for r in rc if r > 0)


def test_shared_system_prompt_is_stored_once():
    B, prompt, requests, own = 16, 1000, 50, 40
    pool = pk.BlockPool(4000)
    seqs = pk.SequenceTables(pool, B)
    root = seqs.add()
    seqs.append_n(root, prompt)
    kids = [seqs.fork(root) for _ in range(requests)]
    for k in kids:
        seqs.append_n(k, own)
    shared = prompt // B                       # full prompt blocks stay shared
    for b in seqs.table(root)[:shared]:
        assert pool.refcount(b) == requests + 1
    used = 4000 - pool.num_free()
    unshared = (requests + 1) * (-(-prompt // B)) + requests * (-(-(own + prompt % B) // B))
    assert used < unshared / 10
    for k in kids:
        seqs.free(k)
    seqs.free(root)
    assert pool.num_free() == 4000
