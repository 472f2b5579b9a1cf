"""Pins for the bitwise write / copy oracle (CPU only)."""

import numpy as np
import pytest

from golden_io import read_kv
from oracle import cache_ops as C


def test_golden_write_slots():
    g = read_kv("write_slots.txt")
    nb, B, d = g["num_blocks"], g["block_size"], g["head_dim"]
    k = np.array(g["k_rows"], np.int16)[:, None, :]          # [T, 1, d]
    v = -k
    kc = np.zeros((nb, 1, B, d), np.int16)
    vc = np.zeros((nb, 1, B, d), np.int16)
    k2, v2 = C.write_kv(k, v, g["slots"], kc, vc)
    want = np.zeros_like(kc)
    for key, row in g["expected_k"].items():
        blk, off = (int(x) for x in key.split(","))
        want[blk, 0, off] = row
    assert np.array_equal(k2, want)
    assert np.array_equal(v2, -want)
    assert np.array_equal(kc, np.zeros_like(kc)), "inputs are not modified"


def test_write_then_gather_returns_each_token_in_order():
    """Writing positions 0..n-1 through a table and reading back gives the rows."""
    rng = np.random.default_rng(0)
    nb, hkv, B, d, n = 20, 3, 4, 5, 37
    table = rng.permutation(nb)[: -(-n // B)]
    k = rng.integers(-30000, 30000, size=(n, hkv, d)).astype(np.int16)
    v = rng.integers(-30000, 30000, size=(n, hkv, d)).astype(np.int16)
    slots = [int(table[p // B]) * B + p % B for p in range(n)]
    kc = np.full((nb, hkv, B, d), 7, np.int16)
    vc = np.full((nb, hkv, B, d), 7, np.int16)
    k2, v2 = C.write_kv(k, v, slots, kc, vc)
    for p in range(n):
        assert np.array_equal(k2[table[p // B], :, p % B], k[p])
        assert np.array_equal(v2[table[p // B], :, p % B], v[p])
    touched = np.zeros((nb, B), bool)
    for s in slots:
        touched[s // B, s % B] = True
    for b in range(nb):
        for o in range(B):
            if not touched[b, o]:
                assert (k2[b, :, o] == 7).all() and (v2[b, :, o] == 7).all()


def test_write_skips_minus_one_and_rejects_duplicates():
    kc = np.zeros((2, 1, 2, 1), np.int16)
    k = np.array([[[5]], [[6]]], np.int16)
    k2, _ = C.write_kv(k, k, [-1, 3], kc, kc)
    assert k2[1, 0, 1, 0] == 6 and int(np.count_nonzero(k2)) == 1
    with pytest.raises(AssertionError):
        C.write_kv(k, k, [2, 2], kc, kc)


def test_copy_blocks_moves_whole_blocks_in_every_cache():
    rng = np.random.default_rng(1)
    caches = [rng.integers(0, 2**31, size=(10, 2, 4, 3)).astype(np.uint32) for _ in range(4)]
    pairs = np.array([[1, 7], [4, 2], [1, 9]])
    out = C.copy_blocks(caches, pairs)
    for c0, c1 in zip(caches, out):
        for b in range(10):
            src = {7: 1, 2: 4, 9: 1}.get(b, b)
            assert np.array_equal(c1[b], c0[src])


def test_copy_blocks_rejects_overlapping_pairs():
    c = np.zeros((4, 1, 1, 1), np.int16)
    with pytest.raises(AssertionError):
        C.copy_blocks([c], [[0, 1], [1, 2]])
    with pytest.raises(AssertionError):
        C.copy_blocks([c], [[0, 3], [1, 3]])


def test_last_token_slot_is_the_slot_the_allocator_gave_that_token():
    """Pinned to the allocator model: after random appends and forks, the slot
    the allocator returned for each sequence's latest append is the slot
    last_token_slots computes from the final table and length."""
    from oracle import allocator as A

    rng = np.random.default_rng(5)
    for B in (1, 4, 16):
        pool = A.BlockPool(400, init_free_order=list(rng.permutation(400)))
        seqs = A.SequenceTables(pool, B)
        ids = [seqs.add() for _ in range(6)]
        latest = {}
        for step in range(120):
            sid = ids[int(rng.integers(len(ids)))]
            if rng.random() < 0.05 and seqs.lens[sid] > 0:
                child = seqs.fork(sid)
                ids.append(child)
                latest[child] = latest[sid]
                continue
            latest[sid], _ = seqs.append(sid)
        live = [s for s in ids if seqs.lens[s] > 0]
        width = max(len(seqs.tables[s]) for s in live)
        tables = np.full((len(live), width), -1, np.int64)
        for i, s in enumerate(live):
            tables[i, :len(seqs.tables[s])] = seqs.tables[s]
        lens = [seqs.lens[s] for s in live]
        got = C.last_token_slots(tables, lens, B)
        want = [latest[s] for s in live]
        # a forked child shares its parent's blocks until it appends: its
        # newest token is the parent's at fork time, in the same slot
        assert list(got) == want


def test_append_token_places_the_new_row_last_in_the_gathered_sequence():
    from oracle import attention as OA

    rng = np.random.default_rng(6)
    nb, hkv, B, d = 30, 2, 4, 3
    kc = rng.integers(-99, 99, (nb, hkv, B, d)).astype(np.int16)
    vc = rng.integers(-99, 99, (nb, hkv, B, d)).astype(np.int16)
    lens = [1, 4, 5, 8, 13]
    perm = rng.permutation(nb)
    tables = np.zeros((len(lens), 4), np.int64)
    tables.flat[:] = perm[:tables.size]
    kn = rng.integers(-99, 99, (len(lens), hkv, d)).astype(np.int16)
    vn = rng.integers(-99, 99, (len(lens), hkv, d)).astype(np.int16)
    k2, v2 = C.append_token(kn, vn, tables, lens, kc, vc)
    for s, n in enumerate(lens):
        for h in range(hkv):
            K = OA.gather_sequence(k2, tables[s], n, h)
            V = OA.gather_sequence(v2, tables[s], n, h)
            K0 = OA.gather_sequence(kc, tables[s], n, h)
            assert np.array_equal(K[-1], kn[s, h]) and np.array_equal(V[-1], vn[s, h])
            assert np.array_equal(K[:-1], K0[:-1])          # earlier rows untouched
    changed = int((k2 != kc).any(axis=3).sum())
    assert changed <= len(lens) * hkv                       # one row per (sequence, KV head)
