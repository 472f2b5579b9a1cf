"""The C++ allocator (through the C ABI) against the hand-worked trace and, bit
for bit, against the oracle allocator on random traces (CPU only)."""

import numpy as np
import pytest

import paged_kv_cache_364_b200 as pk
from golden_io import read_trace
from oracle import allocator as AL
from test_oracle_allocator import OracleBackend, replay_trace


class LibBackend:
    def __init__(self, num_blocks, block_size, order):
        self.pool = pk.BlockPool(num_blocks, order)
        self.seqs = pk.SequenceTables(self.pool, block_size)

    def add(self):
        return self.seqs.add()

    def append(self, sid):
        try:
            slots, pairs = self.seqs.append([sid])
        except pk.OutOfBlocks:
            return "OOM", None
        return slots[0], (pairs[0] if pairs else None)

    def fork(self, sid):
        return self.seqs.fork(sid)

    def free(self, sid):
        self.seqs.free(sid)

    def state(self):
        return {
            "rc": self.pool.refcounts(),
            "free": self.pool.free_list(),
            "tables": {s: self.seqs.table(s) for s in self.seqs.live()},
            "lens": {s: self.seqs.length(s) for s in self.seqs.live()},
        }


def test_library_replays_golden_trace():
    copies = replay_trace(read_trace("allocator_trace.txt"), LibBackend)
    assert copies == [(1, 2), (1, 3), (2, 5)]


@pytest.mark.parametrize("seed", range(8))
def test_random_traces_match_oracle_bit_for_bit(seed):
    rng = np.random.default_rng(1000 + seed)
    nb, B = int(rng.integers(8, 80)), int(rng.choice([1, 2, 4, 16]))
    order = rng.permutation(nb)
    ref = OracleBackend(nb, B, order)
    lib = LibBackend(nb, B, order)
    live = []
    for _ in range(700):
        r = rng.random()
        if r < 0.1 or not live:
            a, b = ref.add(), lib.add()
            assert a == b
            live.append(a)
        elif r < 0.7:
            sid = int(rng.choice(live))
            assert ref.append(sid) == lib.append(sid)
        elif r < 0.85:
            sid = int(rng.choice(live))
            a, b = ref.fork(sid), lib.fork(sid)
            assert a == b
            live.append(a)
        else:
            sid = live.pop(int(rng.integers(len(live))))
            ref.free(sid)
            lib.free(sid)
        assert ref.state() == lib.state()


def test_batched_append_matches_sequential_oracle():
    rng = np.random.default_rng(7)
    nb, B = 200, 16
    order = rng.permutation(nb)
    pool = AL.BlockPool(nb, order)
    ref = AL.SequenceTables(pool, B)
    lp = pk.BlockPool(nb, order)
    lib = pk.SequenceTables(lp, B)
    ids = [ref.add() for _ in range(6)]
    assert [lib.add() for _ in range(6)] == ids
    for _ in range(3):
        kids = [ref.fork(i) for i in ids[:3]]
        assert [lib.fork(i) for i in ids[:3]] == kids
        ids += kids
    for _ in range(40):
        batch = [int(x) for x in rng.choice(ids, size=5, replace=False)]
        want_slots, want_pairs = ref.append_many(batch)
        slots, pairs = lib.append(batch)
        assert slots == want_slots and pairs == want_pairs
        t_slots, t_pairs = lib.append_arrays(batch)
        w_slots, w_pairs = ref.append_many(batch)
        assert t_slots.tolist() == w_slots and [tuple(p) for p in t_pairs.tolist()] == w_pairs
    assert lp.refcounts() == pool.refcount
    assert lp.free_list() == pool.free
    tables, lens = lib.block_tables(ids, max_blocks=20, pad=-7)
    for i, sid in enumerate(ids):
        t = ref.table(sid)
        assert tables[i, : len(t)].tolist() == t
        assert (tables[i, len(t):] == -7).all()
        assert lens[i] == ref.lens[sid]


def test_oom_reports_partial_batch_and_keeps_state():
    lp = pk.BlockPool(2)
    seqs = pk.SequenceTables(lp, 2)
    a, b = seqs.add(), seqs.add()
    seqs.append([a, b])                 # one block each, pool now empty
    before = (lp.refcounts(), lp.free_list(), seqs.table(a), seqs.table(b))
    seqs.append([a])                    # fills block of a
    with pytest.raises(pk.OutOfBlocks) as ei:
        seqs.append([b, a])             # b fits (slot 1 of its block), a needs a block
    assert ei.value.done == 1
    assert seqs.length(a) == 2 and seqs.length(b) == 2
    assert lp.free_list() == [] and lp.refcounts() == before[0]


def test_pool_level_errors():
    lp = pk.BlockPool(4, [3, 2, 1, 0])
    assert lp.alloc() == 0
    with pytest.raises(pk.AllocatorStateError):
        lp.decref([0, 0])
    with pytest.raises(pk.AllocatorStateError):
        lp.incref([2])
    with pytest.raises(pk.AllocatorStateError):
        lp.cow(3)
    assert lp.cow(0) == (0, False)
    lp.incref([0], 2)
    t, copied = lp.cow(0)
    assert copied and t == 1 and lp.refcount(0) == 2 and lp.refcount(1) == 1
    with pytest.raises(ValueError):
        pk.BlockPool(3, [0, 1])
    with pytest.raises(pk.PagedKVError):
        pk.BlockPool(3, [0, 1, 1])


def test_block_tables_into_caller_buffers():
    """block_tables(out=...) fills the given int32 buffers exactly like the
    allocating form, and rejects buffers of the wrong shape or dtype."""
    import pytest
    import torch

    pool = pk.BlockPool(80, np.random.default_rng(4).permutation(80))
    seqs = pk.SequenceTables(pool, 16)
    ids = [seqs.add() for _ in range(4)]
    for i, s in enumerate(ids):
        seqs.append_n(s, 3 + 37 * i)
    want_t, want_l = seqs.block_tables(ids, 12)
    t = torch.full((4, 12), 7, dtype=torch.int32)
    l = torch.full((4,), 7, dtype=torch.int32)
    got_t, got_l = seqs.block_tables(ids, 12, out=(t, l))
    assert got_t is t and got_l is l
    assert torch.equal(t, want_t) and torch.equal(l, want_l)
    with pytest.raises(ValueError):
        seqs.block_tables(ids, 12, out=(torch.empty(4, 11, dtype=torch.int32), l))
    with pytest.raises(ValueError):
        seqs.block_tables(ids, 12, out=(t, torch.empty(4, dtype=torch.int64)))
