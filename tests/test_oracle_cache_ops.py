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
