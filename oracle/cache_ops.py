"""Bitwise cache writes and block copies (oracle; test infrastructure only).

Both operations move stored bits and do no arithmetic on values, so the oracle
works on integer views of the caches (uint16 for fp16/bf16, uint32 for fp32)
and the GPU results must match it bit for bit.

Slot-mapping write ("append")
    A new token at position ``pos`` of a sequence goes into the current
    physical block of that sequence, at offset ``pos % B``; the caller turns
    (block table, position) into a flat slot id ``slot = block * B + offset``
    ([SW] "Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
    Technical Details, "Single Sequence Generation": new tokens fill remaining
    slots of the current physical block; [ML] "49 vLLM / PagedAttention", "The
    block table (the paging idea)", where the append writes the token's K/V
    into the sequence's last block).  Here the slot is given; a slot of -1
    means "skip this token".

Copy-on-write block copy
    On divergence only the diverging block is copied to a new physical block
    ([SW] Technical Details, "Copy-on-Write for Parallel Sampling").  A copy
    moves the whole block -- every KV head, every slot, every element -- and is
    applied to every cache that the block id indexes (K and V of each layer).
"""

from __future__ import annotations

import numpy as np


def write_kv(k, v, slot_mapping, k_cache, v_cache):
    """Return new (k_cache, v_cache) with each token's rows stored in its slot.

    k, v: [T, Hkv, d]; slot_mapping: [T] ints (-1 = skip); caches:
    [NB, Hkv, B, d].  All arrays must share one integer dtype (bit views).
    Slots other than -1 must be distinct and inside the pool.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    num_blocks, _, block_size, _ = k_out.shape
    slots = [int(x) for x in np.asarray(slot_mapping).reshape(-1)]
    live = [s for s in slots if s != -1]
    assert len(set(live)) == len(live), "duplicate slots in one write"
    for t, slot in enumerate(slots):
        if slot == -1:
            continue
        assert 0 <= slot < num_blocks * block_size, "slot outside the pool"
        block, offset = divmod(slot, block_size)
        k_out[block, :, offset, :] = k[t]
        v_out[block, :, offset, :] = v[t]
    return k_out, v_out


def last_token_slots(block_tables, context_lens, block_size: int):
    """Slot of each sequence's newest token, at position ``n_s - 1``.

    The token at position ``pos`` sits in logical block ``pos // B`` of the
    sequence at offset ``pos % B`` ([SW] Technical Details, "Single Sequence
    Generation"; [ML] "The block table (the paging idea)"), so its slot is
    ``table[s][pos // B] * B + pos % B`` with ``pos = context_lens[s] - 1``.
    """
    tables = np.asarray(block_tables)
    out = []
    for s, n in enumerate(np.asarray(context_lens).reshape(-1)):
        pos = int(n) - 1
        assert pos >= 0, "a sequence needs at least one token"
        out.append(int(tables[s, pos // block_size]) * block_size + pos % block_size)
    return np.array(out, dtype=np.int64)


def append_token(k_new, v_new, block_tables, context_lens, k_cache, v_cache):
    """The cache update of a fused append + decode step: each sequence's new
    rows ``k_new[s]``, ``v_new[s]`` stored at its newest position."""
    B = np.asarray(k_cache).shape[2]
    return write_kv(k_new, v_new, last_token_slots(block_tables, context_lens, B), k_cache, v_cache)


def copy_blocks(caches, src_dst_pairs):
    """Return copies of every cache with ``cache[dst] = cache[src]`` per pair.

    caches: list of [NB, ...] integer arrays; src_dst_pairs: [P, 2] ints.
    Destinations are distinct and disjoint from sources (the allocator hands
    out fresh blocks as destinations), so the copies commute.
    """
    pairs = [(int(a), int(b)) for a, b in np.asarray(src_dst_pairs).reshape(-1, 2)]
    srcs = {a for a, _ in pairs}
    dsts = [b for _, b in pairs]
    assert len(set(dsts)) == len(dsts), "a destination block appears twice"
    assert not (srcs & set(dsts)), "a destination block is also a source"
    out = []
    for cache in caches:
        c = np.array(cache, copy=True)
        for src, dst in pairs:
            c[dst] = cache[src]
        out.append(c)
    return out
