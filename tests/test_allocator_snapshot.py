"""Pool statistics and checkpoint / resume of the host allocator (CPU only).

``pa_alloc_stats`` is checked against counts derived from the oracle
allocator's state.  ``pa_seqs_snapshot`` is parsed independently and compared
field by field with the oracle's pool and tables; a restored table set must
continue a random trace exactly as the original and the oracle do; damaged
snapshots are refused.
"""

import struct

import numpy as np
import pytest

import paged_kv_cache_364_b200 as pk
from oracle import allocator as AL


def random_ops(rng, n_ops, live):
    """Yield (kind, arg) operations over the ids in ``live`` (updated by the caller)."""
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.1 or not live:
            yield "add", None
        elif r < 0.65:
            yield "append", int(rng.choice(live))
        elif r < 0.8:
            yield "fork", int(rng.choice(live))
        else:
            yield "free", int(live[int(rng.integers(len(live)))])


def apply(op, arg, seqs, live, oom_error):
    if op == "add":
        sid = seqs.add()
        live.append(sid)
        return sid
    if op == "append":
        try:
            slots, pairs = seqs.append([arg]) if isinstance(seqs, pk.SequenceTables) else seqs.append(arg)
        except oom_error:
            return "OOM"
        if isinstance(seqs, pk.SequenceTables):
            return slots[0], (tuple(pairs[0]) if pairs else None)
        return slots, (tuple(pairs) if pairs is not None else None)
    if op == "fork":
        child = seqs.fork(arg)
        live.append(child)
        return child
    seqs.free(arg)
    live.remove(arg)
    return None


def lib_state(seqs):
    return {"rc": seqs.pool.refcounts(), "free": seqs.pool.free_list(),
            "tables": {s: seqs.table(s) for s in seqs.live()}, "lens": {s: seqs.length(s) for s in seqs.live()}}


def oracle_state(seqs):
    return {"rc": list(seqs.pool.refcount), "free": list(seqs.pool.free),
            "tables": {s: list(t) for s, t in seqs.tables.items()}, "lens": dict(seqs.lens)}


def make_pair(seed):
    rng = np.random.default_rng(seed)
    nb, B = int(rng.integers(8, 60)), int(rng.choice([1, 4, 16]))
    order = rng.permutation(nb)
    return rng, nb, B, pk.SequenceTables(pk.BlockPool(nb, order), B), AL.SequenceTables(AL.BlockPool(nb, order), B)


@pytest.mark.parametrize("seed", range(5))
def test_stats_match_the_oracle_counts(seed):
    rng, nb, B, lib, ref = make_pair(300 + seed)
    live_l, live_r = [], []
    for op, arg in random_ops(rng, 300, live_r):
        a = apply(op, arg, ref, live_r, AL.OutOfBlocks)
        b = apply(op, arg, lib, live_l, pk.OutOfBlocks)
        assert a == b
        rc = ref.pool.refcount
        assert lib.pool.stats() == {"num_blocks": nb, "free_blocks": len(ref.pool.free),
                                    "used_blocks": sum(c > 0 for c in rc), "shared_blocks": sum(c > 1 for c in rc),
                                    "references": sum(rc)}


def parse_snapshot(data):
    """The documented layout, read independently of the library."""
    w = struct.unpack(f"={len(data) // 4}i", data)
    magic, version, nb, B, next_id, n_free, n_seqs = w[:7]
    at = 7
    free = list(w[at:at + n_free])
    at += n_free
    rc = list(w[at:at + nb])
    at += nb
    tables, lens = {}, {}
    for _ in range(n_seqs):
        sid, n, k = w[at:at + 3]
        tables[sid] = list(w[at + 3:at + 3 + k])
        lens[sid] = n
        at += 3 + k
    assert at == len(w)
    return dict(magic=magic & 0xFFFFFFFF, version=version, nb=nb, B=B, next_id=next_id, free=free, rc=rc,
                tables=tables, lens=lens)


@pytest.mark.parametrize("seed", range(5))
def test_snapshot_layout_holds_the_oracle_state(seed):
    rng, nb, B, lib, ref = make_pair(400 + seed)
    live_l, live_r = [], []
    issued = 0                                 # ids handed out by add and fork
    for op, arg in random_ops(rng, 250, live_r):
        assert apply(op, arg, ref, live_r, AL.OutOfBlocks) == apply(op, arg, lib, live_l, pk.OutOfBlocks)
        issued += op in ("add", "fork")
    snap = parse_snapshot(lib.snapshot())
    assert snap["magic"] == 0x564B4150 and snap["version"] == 1 and snap["nb"] == nb and snap["B"] == B
    want = oracle_state(ref)
    assert snap["free"] == want["free"] and snap["rc"] == want["rc"]
    assert snap["tables"] == want["tables"] and snap["lens"] == want["lens"]
    assert snap["next_id"] == issued


@pytest.mark.parametrize("seed", range(6))
def test_restored_tables_continue_like_the_original(seed):
    rng, nb, B, lib, ref = make_pair(500 + seed)
    live_l, live_r = [], []
    for op, arg in random_ops(rng, 200, live_r):
        assert apply(op, arg, ref, live_r, AL.OutOfBlocks) == apply(op, arg, lib, live_l, pk.OutOfBlocks)
    data = lib.snapshot()
    back = pk.SequenceTables.restore(data)
    assert back.snapshot() == data and back.block_size == B
    live_b = list(live_l)
    for op, arg in random_ops(rng, 200, live_r):
        a = apply(op, arg, ref, live_r, AL.OutOfBlocks)
        assert apply(op, arg, lib, live_l, pk.OutOfBlocks) == a
        assert apply(op, arg, back, live_b, pk.OutOfBlocks) == a
    assert lib_state(back) == lib_state(lib) == oracle_state(ref)
    assert back.snapshot() == lib.snapshot()


def damaged(data, word, value):
    w = list(struct.unpack(f"={len(data) // 4}i", data))
    w[word] = value
    return struct.pack(f"={len(w)}i", *w)


def test_damaged_snapshots_are_refused():
    pool = pk.BlockPool(6)
    seqs = pk.SequenceTables(pool, 4)
    a = seqs.add()
    seqs.append_n(a, 5)                        # blocks 0, 1
    b = seqs.fork(a)                           # both shared
    seqs.append([b])                           # b copies block 1 -> 2: counts [2, 1, 1, 0, 0, 0]
    data = seqs.snapshot()
    pk.SequenceTables.restore(data)            # the intact snapshot is accepted
    n_free = struct.unpack_from("=i", data, 20)[0]
    rc0 = 7 + n_free                           # word index of block 0's count
    bad = [
        data[:-4],                             # truncated
        data + b"\0\0\0\0",                    # trailing word
        data[:6],                              # not whole words
        damaged(data, 0, 0x12345678),          # magic
        damaged(data, 1, 2),                   # version
        damaged(data, 3, 0),                   # block size
        damaged(data, 7, 0),                   # free pool names a block in use
        damaged(data, rc0, 0),                 # count 0 for a block in a table and not free
        damaged(data, rc0, 1),                 # block 0 is in both tables but counted once
        damaged(data, rc0 + 3, 1),             # block 3 counted but also in the free pool
    ]
    for blob in bad:
        with pytest.raises(pk.PagedKVError, match="snapshot"):
            pk.SequenceTables.restore(blob)


def test_snapshot_size_query_and_capacity(lib):
    import ctypes

    seqs = pk.SequenceTables(pk.BlockPool(4), 2)
    seqs.append_n(seqs.add(), 3)
    n = ctypes.c_uint64()
    assert lib.pa_seqs_snapshot(seqs._h, None, 0, ctypes.byref(n)) == 0
    assert n.value == 4 * (7 + 2 + 4 + 3 + 2)  # header, free [2], counts [4], one table of 2 blocks
    small = ctypes.create_string_buffer(int(n.value) - 4)
    assert lib.pa_seqs_snapshot(seqs._h, small, n.value - 4, ctypes.byref(n)) == pk._lib.PA_ERR_ARG
