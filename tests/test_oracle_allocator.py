"""Pins for the allocator oracle (CPU only).

Checked against a hand-worked trace, against invariants the pages state, and
end to end: appends, forks and copy-on-write driven through the bitwise write
and copy oracles must leave every live sequence reading back exactly the
tokens it was given.
"""

import numpy as np
import pytest

from golden_io import read_trace
from oracle import allocator as AL
from oracle import attention as AT
from oracle import cache_ops as C


class OracleBackend:
    def __init__(self, num_blocks, block_size, order):
        self.pool = AL.BlockPool(num_blocks, order)
        self.seqs = AL.SequenceTables(self.pool, block_size)

    def add(self):
        return self.seqs.add()

    def append(self, sid):
        try:
            return self.seqs.append(sid)
        except AL.OutOfBlocks:
            return "OOM", None

    def fork(self, sid):
        return self.seqs.fork(sid)

    def free(self, sid):
        self.seqs.free(sid)

    def state(self):
        return {
            "rc": list(self.pool.refcount),
            "free": list(self.pool.free),
            "tables": {s: list(t) for s, t in self.seqs.tables.items()},
            "lens": dict(self.seqs.lens),
        }


def replay_trace(ops, make_backend):
    be = None
    copies = []
    for op in ops:
        kind = op[0]
        if kind == "pool":
            be = make_backend(op[1], op[2], op[3])
        elif kind == "add":
            assert be.add() == op[1]
        elif kind == "append":
            slot, pair = be.append(op[1])
            assert slot == op[2], op
            assert (tuple(pair) if pair is not None else None) == op[3], op
            if pair is not None:
                copies.append(tuple(pair))
        elif kind == "fork":
            assert be.fork(op[1]) == op[2]
        elif kind == "free":
            be.free(op[1])
        elif kind == "state":
            st = be.state()
            want = op[1]
            assert st["rc"] == want["rc"]
            assert st["free"] == want["free"]
            assert st["tables"] == want["tables"]
            assert st["lens"] == want["lens"]
    return copies


def test_golden_trace():
    copies = replay_trace(read_trace("allocator_trace.txt"), OracleBackend)
    assert copies == [(1, 2), (1, 3), (2, 5)]


def _check_invariants(seqs: AL.SequenceTables):
    pool = seqs.pool
    B = seqs.block_size
    # every reference is a table entry, and vice versa
    counts = [0] * pool.num_blocks
    for t in seqs.tables.values():
        for b in t:
            counts[b] += 1
    assert counts == pool.refcount
    # the free pool holds exactly the unreferenced blocks, once each
    assert sorted(pool.free) == [b for b in range(pool.num_blocks) if pool.refcount[b] == 0]
    assert len(pool.free) == pool.num_blocks - sum(1 for r in pool.refcount if r > 0)
    # waste bounded by the last block: blocks per sequence = ceil(len / B)
    for sid, t in seqs.tables.items():
        assert len(t) == -(-seqs.lens[sid] // B)


@pytest.mark.parametrize("seed", range(6))
def test_random_traces_keep_invariants(seed):
    rng = np.random.default_rng(seed)
    nb, B = 64, 4
    pool = AL.BlockPool(nb, rng.permutation(nb))
    seqs = AL.SequenceTables(pool, B)
    live = [seqs.add()]
    for _ in range(600):
        r = rng.random()
        if r < 0.65 and live:
            sid = int(rng.choice(live))
            try:
                seqs.append(sid)
            except AL.OutOfBlocks:
                victim = live.pop(int(rng.integers(len(live))))
                seqs.free(victim)
        elif r < 0.8 and live:
            live.append(seqs.fork(int(rng.choice(live))))
        elif r < 0.9 and len(live) > 1:
            seqs.free(live.pop(int(rng.integers(len(live)))))
        else:
            live.append(seqs.add())
        _check_invariants(seqs)


def test_errors_leave_state_unchanged():
    pool = AL.BlockPool(2, [1, 0])
    seqs = AL.SequenceTables(pool, 2)
    a = seqs.add()
    for _ in range(4):
        seqs.append(a)
    snap = (list(pool.refcount), list(pool.free), seqs.table(a), seqs.lens[a])
    with pytest.raises(AL.OutOfBlocks):
        seqs.append(a)
    assert snap == (list(pool.refcount), list(pool.free), seqs.table(a), seqs.lens[a])
    with pytest.raises(AL.AllocatorStateError):
        pool.decref([0, 0])
    with pytest.raises(AL.AllocatorStateError):
        pool.incref([5])
    assert snap == (list(pool.refcount), list(pool.free), seqs.table(a), seqs.lens[a])


def test_one_block_copy_per_branching_event():
    """Forking n ways and diverging copies n-1 blocks (the last writer keeps it)."""
    for n in (2, 3, 8):
        pool = AL.BlockPool(64)
        seqs = AL.SequenceTables(pool, 16)
        p = seqs.add()
        for _ in range(20):                   # one full block + 4 tokens
            seqs.append(p)
        kids = [seqs.fork(p) for _ in range(n - 1)]
        pairs = [seqs.append(s)[1] for s in [p] + kids]
        assert sum(x is not None for x in pairs) == n - 1
        assert pool.refcount[seqs.table(p)[0]] == n   # the full block stays shared


def test_sharing_workload_counts():
    """16 prompts x 1000 tokens, 8 samples each, block size 16.

    Hand count: 1000 = 62 * 16 + 8, so 63 blocks per prompt, the last one
    holding 8 tokens; after forking, every prompt block has count 8; each
    sample's first write into the partial block copies it except the last
    writer's, so 7 copies per prompt and 112 in all.
    """
    B, prompts, samples = 16, 16, 8
    pool = AL.BlockPool(16 * 63 + 16 * 7 + 16 * 8 * 20)
    seqs = AL.SequenceTables(pool, B)
    groups = []
    for _ in range(prompts):
        p = seqs.add()
        for _ in range(1000):
            seqs.append(p)
        assert len(seqs.table(p)) == 63
        groups.append([p] + [seqs.fork(p) for _ in range(samples - 1)])
    for g in groups:
        for b in seqs.table(g[0]):
            assert pool.refcount[b] == 8
    n_copies = 0
    for g in groups:
        for sid in g:
            _, pair = seqs.append(sid)
            n_copies += pair is not None
    assert n_copies == 112


@pytest.mark.parametrize("seed", range(4))
def test_tables_write_and_copy_read_back_every_token(seed):
    """End to end on the oracles: fork / append / CoW / free, then gather.

    Each token gets a unique id written as its K row; after every step the
    gathered logical rows of each live sequence equal its own history.
    """
    rng = np.random.default_rng(100 + seed)
    nb, B, d = 48, 4, 2
    pool = AL.BlockPool(nb, rng.permutation(nb))
    seqs = AL.SequenceTables(pool, B)
    kc = np.zeros((nb, 1, B, d), np.int32)
    history = {}
    next_tok = [1]

    def append(sid):
        slot, pair = seqs.append(sid)
        nonlocal kc
        if pair is not None:
            (kc,) = C.copy_blocks([kc], np.array([pair]))
        tok = next_tok[0]
        next_tok[0] += 1
        row = np.array([[[tok, -tok]]], np.int32)
        kc, _ = C.write_kv(row, row, [slot], kc, kc)
        history[sid].append(tok)

    first = seqs.add()
    history[first] = []
    live = [first]
    for step in range(400):
        r = rng.random()
        try:
            if r < 0.7:
                append(int(rng.choice(live)))
            elif r < 0.85 and len(live) < 8:
                parent = int(rng.choice(live))
                child = seqs.fork(parent)
                history[child] = list(history[parent])
                live.append(child)
            elif len(live) > 1:
                victim = live.pop(int(rng.integers(len(live))))
                seqs.free(victim)
                del history[victim]
        except AL.OutOfBlocks:
            victim = live.pop(0) if len(live) > 1 else None
            if victim is not None:
                seqs.free(victim)
                del history[victim]
        for sid in live:
            n = seqs.lens[sid]
            if n == 0:
                continue
            rows = AT.gather_sequence(kc, seqs.table(sid), n, 0)
            assert rows[:, 0].astype(np.int64).tolist() == history[sid]
