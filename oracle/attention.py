"""Decode attention over a paged KV cache, float64 (oracle; test infrastructure only).

What is computed
----------------
The cache is cut into fixed-size physical blocks of ``B`` token slots, and a
per-sequence block table maps logical block ``i`` (token positions
``i*B .. i*B+B-1``) to a physical block id anywhere in the pool
([SW] "Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention",
Technical Details, "Core Architecture"; [ML] "49 vLLM / PagedAttention",
"The idea and the mechanism").  Paging "does not change transformer math"
([PV] "PagedAttention: How Virtual Memory Paging Solved LLM KV Cache Waste",
Key points, "Engineering insight"; [ML] "Connections", the FlashAttention
entry): the result of decode attention over the paged cache is exactly the
result of ordinary single-query softmax attention over the sequence's
contiguous K and V.  So the oracle is that definition written out:

  1. rebuild the sequence's contiguous ``K_s`` / ``V_s`` ([n_s, d]) by walking
     its block table (``gather_sequence``);
  2. upcast the stored values exactly to float64;
  3. ``out = softmax(scale * K_s @ q) @ V_s`` with the max-subtracted softmax.

Grouped-query attention: query head ``h`` reads KV head ``h // (Hq // Hkv)``
(contiguous groups).  The pages do not fix the mapping; this is the plainest
reading.

Layout conventions (the pages give none): ``k_cache`` / ``v_cache`` are
``[num_blocks, Hkv, B, d]``; ``block_tables`` is ``[batch, max_blocks]``;
``context_lens`` is ``[batch]`` and counts every token attended, including the
one written in the same decode step.

Split-context helpers (``partial_state`` / ``lse_merge``) exist only so a test
can pin the identity "merging per-chunk partial softmax states equals the
unsplit result"; the oracle's own ``paged_decode`` never splits.
"""

from __future__ import annotations

import numpy as np


def to_f64(x) -> np.ndarray:
    """Exact upcast of stored values to float64.

    Accepts numpy arrays (float16/float32/float64) or torch tensors (any float
    dtype including bfloat16, on any device); every fp16/bf16/fp32 value is
    exactly representable in float64, so this step adds no rounding.
    """
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _as_int_array(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


def gather_sequence(cache, table_row, n_tokens: int, kv_head: int) -> np.ndarray:
    """Contiguous ``[n_tokens, d]`` rows of one sequence, rebuilt from its pages.

    Logical block ``i`` of the sequence lives in physical block
    ``table_row[i]`` ("a Block Table maintains a mapping from contiguous Logical
    Blocks ... to scattered Physical Blocks", [SW] Technical Details, "Core
    Architecture").  Only the first ``ceil(n_tokens / B)`` table entries are
    read, and the unfilled slots of the last block are dropped ("memory waste is
    strictly bounded to the unfilled slots of the last block", [SW] "Single
    Sequence Generation").  Returns float64.
    """
    block_size = cache.shape[2]
    n_blocks = -(-n_tokens // block_size)
    pages = [to_f64(cache[int(table_row[i]), kv_head]) for i in range(n_blocks)]
    if not pages:
        return np.zeros((0, cache.shape[3]), np.float64)
    return np.concatenate(pages, axis=0)[:n_tokens]


def softmax(scores: np.ndarray) -> np.ndarray:
    """Textbook max-subtracted softmax of a 1-D float64 vector."""
    z = scores - scores.max()
    e = np.exp(z)
    return e / e.sum()


def contiguous_attention(q, K, V, scale: float) -> np.ndarray:
    """Single-query attention ``softmax(scale * K q) V`` over contiguous K, V.

    q: [d]; K, V: [n, d]; all float64; n >= 1.
    """
    s = scale * (K @ q)
    return softmax(s) @ V


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """Decode attention for a batch over a paged cache, float64 ``[batch, Hq, d]``.

    q: [batch, Hq, d]; k_cache, v_cache: [NB, Hkv, B, d]; block_tables:
    [batch, max_blocks] ints; context_lens: [batch] ints >= 1.
    Works per (sequence, KV head) so memory stays bounded for large pools.
    """
    qf = to_f64(q)
    tables = _as_int_array(block_tables)
    lens = _as_int_array(context_lens)
    batch, n_q_heads, d = qf.shape
    n_kv_heads = k_cache.shape[1]
    assert n_q_heads % n_kv_heads == 0, "query heads must be a multiple of KV heads"
    group = n_q_heads // n_kv_heads
    out = np.empty((batch, n_q_heads, d), np.float64)
    for s in range(batch):
        n = int(lens[s])
        assert n >= 1, "a decode step attends over at least the token it wrote"
        for hk in range(n_kv_heads):
            K = gather_sequence(k_cache, tables[s], n, hk)
            V = gather_sequence(v_cache, tables[s], n, hk)
            for j in range(group):
                h = hk * group + j
                out[s, h] = contiguous_attention(qf[s, h], K, V, scale)
    return out


def paged_decode_rows(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                      rows) -> np.ndarray:
    """``paged_decode`` restricted to the listed sequences (rows of the batch).

    Used to check sampled outputs of a full-size launch one sequence at a time.
    Returns ``[len(rows), Hq, d]`` float64.
    """
    rows = [int(r) for r in rows]
    tables = _as_int_array(block_tables)
    lens = _as_int_array(context_lens)
    qs = to_f64(q)[rows]
    return paged_decode(qs, k_cache, v_cache, tables[rows], lens[rows], scale)


# --- split-context identity (pins the merge the GPU path performs) -----------

def partial_state(q, K, V, scale: float):
    """Unnormalised softmax state of one chunk of keys: (m, l, acc).

    m = max_j s_j, l = sum_j exp(s_j - m), acc = sum_j exp(s_j - m) V_j, with
    s_j = scale * q . K_j.  float64.
    """
    s = scale * (K @ q)
    m = s.max()
    e = np.exp(s - m)
    return m, e.sum(), e @ V


def lse_merge(states) -> np.ndarray:
    """Combine chunk states into the attention output.

    M = max_p m_p;  L = sum_p l_p exp(m_p - M);  out = sum_p exp(m_p - M) acc_p / L.
    """
    ms = np.array([st[0] for st in states], np.float64)
    M = ms.max()
    w = np.exp(ms - M)
    L = sum(wp * st[1] for wp, st in zip(w, states))
    acc = sum(wp * st[2] for wp, st in zip(w, states))
    return acc / L


# --- prefill: several new query tokens per sequence ---------------------------
#
# During prefill a sequence's prompt tokens are placed into logical blocks that
# map to arbitrary physical blocks ([SW] Technical Details, "Single Sequence
# Generation"), and a shared system prompt's blocks can be stored once and
# referenced by every request so that it is not prefilled again ([ML]
# "Questions worth asking", the shared-prompt question).  A prefill step then
# attends the sequence's new tokens over everything before them: its cached
# prefix (possibly shared) and the new tokens up to and including itself.
#
# Reading (the pages give no interface): the new tokens' K/V are written into
# the cache first, as for decode, so ``context_lens[s] = n_s`` counts them; the
# new tokens are the last ``q_len_s`` positions of the sequence, i.e. query row
# ``i`` of sequence ``s`` sits at position ``n_s - q_len_s + i`` and attends
# keys ``0 .. n_s - q_len_s + i`` (causal within the new tokens, the whole
# prefix visible).  Query rows of all sequences are packed: sequence ``s`` owns
# rows ``query_start[s] .. query_start[s+1] - 1``.

def causal_attention(Q, K, V, scale: float, first_pos: int) -> np.ndarray:
    """Rows of ``Q`` ([m, d]) at positions ``first_pos .. first_pos + m - 1``
    over contiguous ``K``, ``V`` ([n, d]); row i sees keys ``0 .. first_pos + i``."""
    out = np.empty((Q.shape[0], V.shape[1]), np.float64)
    for i in range(Q.shape[0]):
        p = first_pos + i
        out[i] = contiguous_attention(Q[i], K[: p + 1], V[: p + 1], scale)
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale: float,
                  seqs=None) -> np.ndarray:
    """Prefill attention over a paged cache, float64 ``[T, Hq, d]``.

    q: [T, Hq, d] packed query rows; query_start: [batch + 1] ints,
    nondecreasing, ``query_start[0] = 0``; ``0 <= q_len_s <= context_lens[s]``.
    With ``seqs`` given, only those sequences' rows are computed and returned
    (in the order listed), for sampled checks of large launches.
    """
    qf = to_f64(q)
    tables = _as_int_array(block_tables)
    lens = _as_int_array(context_lens)
    starts = _as_int_array(query_start)
    n_q_heads, d = qf.shape[1], qf.shape[2]
    n_kv_heads = k_cache.shape[1]
    assert n_q_heads % n_kv_heads == 0, "query heads must be a multiple of KV heads"
    group = n_q_heads // n_kv_heads
    batch = len(lens)
    assert starts[0] == 0 and all(starts[s] <= starts[s + 1] for s in range(batch))
    order = range(batch) if seqs is None else [int(s) for s in seqs]
    pieces = []
    for s in order:
        n = int(lens[s])
        r0, r1 = int(starts[s]), int(starts[s + 1])
        m = r1 - r0
        assert 0 <= m <= n, "a sequence's new tokens are part of its context"
        block = np.empty((m, n_q_heads, d), np.float64)
        for hk in range(n_kv_heads):
            K = gather_sequence(k_cache, tables[s], n, hk)
            V = gather_sequence(v_cache, tables[s], n, hk)
            for j in range(group):
                h = hk * group + j
                block[:, h] = causal_attention(qf[r0:r1, h], K, V, scale, n - m)
        pieces.append(block)
    if not pieces:
        return np.zeros((0, n_q_heads, d), np.float64)
    return np.concatenate(pieces, axis=0)
