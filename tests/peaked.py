"""Inputs whose softmax is peaked and whose running maximum moves far.

The N(0, 1) workloads keep base-2 scores within about +-6, so the online
softmax's running maximum hardly moves after the first keys.  The inputs here
put the kernels where it does: rising scores (the maximum grows on every page
and every 64-key tile), falling scores, a staircase, a spike on the newest
key, a dominant key in the middle, steps just under the prefill kernel's
rescale threshold (a tile maximum 8 above the running one in base 2, i.e.
weights of 2^8), a wide random spread and a flat row.  The exact softmax is
still what must come out ("PagedAttention: How Virtual Memory Paging Solved
LLM KV Cache Waste", Key points: paging leaves the attention math unchanged).

Construction: every query head h reads one pattern column c(h) of K -- its q
row is zero except q[c(h)] = QV, a power of two -- and column c of K carries,
for the token at position j of a sequence of length n, the value
S2_c(j, n) / (QV * scale * log2 e) cast to the cache dtype.  The score of a
key is then QV times that stored value, which every kernel forms without
rounding (one non-zero product, exact in fp32); the oracle gets the same cast
tensors.  |S2| stays below 2^10, so a kernel's fp32 rounding of a scaled score
is at most 2^-15 (base 2), which the tests' precision bound accounts for.
Which column a head reads shifts with its KV head, so the heads of one group,
and the groups of one sequence, see different patterns.
"""

from __future__ import annotations

import math

import numpy as np
import torch

LOG2E = 1.0 / math.log(2.0)
QV = 8.0
S2_CAP = 950.0
PATTERNS = ("rise", "fall", "steps", "last_key", "near_threshold", "wide_random", "dominant_mid", "flat")


def target_scores(pattern: str, n: int, rng: np.random.Generator, cap: float = S2_CAP) -> np.ndarray:
    """Intended base-2 scaled scores of positions 0..n-1 of one sequence
    (|score| <= cap, except "near_threshold", which stays below 48)."""
    j = np.arange(n, dtype=np.float64)
    slope = min(4.5, cap / max(n - 1, 1))
    if pattern == "rise":              # the maximum grows with every key
        s = slope * j
    elif pattern == "fall":            # the first key is the maximum
        s = -slope * j
    elif pattern == "steps":           # jumps every 97 keys, flat in between
        step = min(40.0, cap * 97.0 / max(n, 1))
        s = step * np.floor(j / 97.0)
    elif pattern == "last_key":        # the newest token dominates
        s = rng.standard_normal(n)
        s[-1] = cap
    elif pattern == "near_threshold":  # rises 7.9 per 64 keys for 6 tiles, then drops
        s = 7.9 * (np.floor(j / 64.0) % 7) + 0.1 * rng.standard_normal(n)
    elif pattern == "wide_random":
        s = np.clip(cap / 4.0 * rng.standard_normal(n), -cap, cap)
    elif pattern == "dominant_mid":    # one key far above the rest
        s = rng.standard_normal(n)
        s[n // 3] = cap
    elif pattern == "flat":            # equal scores: the mean of V
        s = np.full(n, 3.0)
    else:
        raise KeyError(pattern)
    return s


def pattern_column(h: int, group: int, n_patterns: int = len(PATTERNS)) -> int:
    """K column (= pattern index) read by query head h."""
    return (h + h // group) % n_patterns


def column_values(lens, scale: float, dtype, seed: int, max_tokens: int, cap: float = S2_CAP) -> torch.Tensor:
    """[batch, max_tokens, P] float32: the K value of every pattern column at
    every position of every sequence (zero past a sequence's length), already
    rounded to ``dtype``."""
    rng = np.random.default_rng(seed)
    c2 = scale * LOG2E
    vals = np.zeros((len(lens), max_tokens, len(PATTERNS)), np.float64)
    for s, n in enumerate(lens):
        n = int(n)
        for c, name in enumerate(PATTERNS):
            vals[s, :n, c] = target_scores(name, n, rng, cap) / (QV * c2)
    return torch.from_numpy(vals).to(dtype).float()


def fill_cache(k_cache: torch.Tensor, tables: np.ndarray, lens, vals: torch.Tensor):
    """Write column values into the K pages of each sequence (every KV head):
    position j of sequence s sits in row j % B of its logical block j // B."""
    nb_, hkv, B, d = k_cache.shape
    P = vals.shape[2]
    for s, n in enumerate(lens):
        nblk = -(-int(n) // B)
        if nblk == 0:
            continue
        ids = torch.from_numpy(np.ascontiguousarray(tables[s, :nblk]).astype(np.int64)).to(k_cache.device)
        page = vals[s, :nblk * B].reshape(nblk, 1, B, P).to(k_cache.dtype).to(k_cache.device)
        k_cache[ids, :, :, :P] = page.expand(nblk, hkv, B, P)


def set_queries(q: torch.Tensor, group: int):
    """Every row of q [rows, Hq, d]: zero except QV at its head's pattern column."""
    q.zero_()
    for h in range(q.shape[1]):
        q[:, h, pattern_column(h, group)] = QV


def score_max(vals: torch.Tensor, scale: float) -> float:
    """Largest |base-2 scaled score| any key produces."""
    return float(vals.abs().max()) * QV * scale * LOG2E


def rounding_bound(s2max: float, vmax: float) -> float:
    """Output error that an fp32 rounding of each scaled score can cause:
    each score off by at most half an ulp of s2max (base 2) changes each
    normalised weight by a relative 2 ln2 times that, and the output moves by
    at most that times max |v - out| <= 2 max |v|."""
    if s2max <= 0:
        return 0.0
    half_ulp = 2.0 ** (math.floor(math.log2(s2max)) - 24)
    return 4.0 * math.log(2.0) * half_ulp * vmax


def tiles_that_grow(vals_row: np.ndarray, scale: float, n_visible: int, col: int, tile: int = 64,
                    threshold: float = 8.0) -> int:
    """How many key tiles after the first raise the running maximum by more
    than ``threshold`` (base 2) for a query row that sees keys 0..n_visible-1
    of one pattern column: the tiles where a lazily rescaled online softmax
    must rescale its accumulator."""
    s2 = vals_row[:n_visible, col].astype(np.float64) * QV * scale * LOG2E
    m, grows = -np.inf, 0
    for t0 in range(0, n_visible, tile):
        mt = s2[t0:t0 + tile].max()
        if mt > m + threshold:
            grows += t0 > 0
            m = mt
    return grows
