"""Pins for the float64 prefill oracle (CPU only).

A prefill row at position p attends keys 0..p of its sequence.  Each test
below fails for a plausible mistake: a hand-worked fixture with exact weights
and a zero-query closed form (wrong alignment of new tokens to positions, a
dropped or extra key), agreement with the decode oracle for one new token,
with torch's causal scaled_dot_product_attention for a full prompt (wrong
mask direction, wrong scale), chunking invariance (prefix handling), paging
invariance (table walk), and a pure-Python brute force.
"""

import math

import numpy as np
import pytest
import torch

from golden_io import read_kv
from oracle import attention as A


def _paged(seqs_k, seqs_v, block_size, rng, extra_blocks=3):
    """Scatter per-sequence contiguous [Hkv, n, d] K/V into a shuffled paged pool."""
    hkv, _, d = seqs_k[0].shape
    nblk = [-(-k.shape[1] // block_size) for k in seqs_k]
    nb = sum(nblk) + extra_blocks
    perm = rng.permutation(nb)
    kc = np.full((nb, hkv, block_size, d), np.nan)
    vc = np.full((nb, hkv, block_size, d), np.nan)
    width = max(nblk)
    tables = np.full((len(seqs_k), width), -1, np.int64)
    i = 0
    for s, (k, v) in enumerate(zip(seqs_k, seqs_v)):
        for b in range(nblk[s]):
            blk = int(perm[i])
            i += 1
            tables[s, b] = blk
            rows = slice(b * block_size, min((b + 1) * block_size, k.shape[1]))
            m = rows.stop - rows.start
            kc[blk, :, :m] = k[:, rows]
            vc[blk, :, :m] = v[:, rows]
    return kc, vc, tables


def _problem(rng, lens, qlens, hq, hkv, d, block_size=4):
    ks = [rng.standard_normal((hkv, n, d)) for n in lens]
    vs = [rng.standard_normal((hkv, n, d)) for n in lens]
    kc, vc, tables = _paged(ks, vs, block_size, rng)
    starts = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int64)
    q = rng.standard_normal((int(starts[-1]), hq, d))
    return q, kc, vc, tables, np.array(lens), starts, ks, vs


def test_golden_prefill_rational():
    g = read_kv("prefill_rational.txt")
    B, d, nb = g["block_size"], g["head_dim"], g["num_blocks"]
    kc = np.full((nb, 1, B, d), np.nan)
    vc = np.full((nb, 1, B, d), np.nan)
    for s, (ws, vrows) in enumerate(zip(g["weights"], g["v_rows"])):
        for pos, (w, v) in enumerate(zip(ws, vrows)):
            blk = g["block_tables"][s][pos // B]
            kc[blk, 0, pos % B] = [math.log(w), 0.0]
            vc[blk, 0, pos % B] = v
    q = np.array(g["q"], np.float64)[:, None, :]
    out = A.paged_prefill(q, kc, vc, np.array(g["block_tables"]), np.array(g["context_lens"]),
                          np.array(g["query_start"]), g["scale"])
    np.testing.assert_allclose(out[:, 0], np.array(g["expected_out"]), rtol=0, atol=1e-12)


def test_zero_query_gives_the_running_mean_of_visible_values():
    rng = np.random.default_rng(1)
    lens, qlens = [9, 6, 13], [4, 6, 1]
    q, kc, vc, tables, lens_a, starts, ks, vs = _problem(rng, lens, qlens, 2, 1, 5)
    out = A.paged_prefill(np.zeros_like(q), kc, vc, tables, lens_a, starts, 0.3)
    for s, (n, m) in enumerate(zip(lens, qlens)):
        for i in range(m):
            p = n - m + i
            want = vs[s][0, : p + 1].mean(axis=0)
            for h in range(2):
                np.testing.assert_allclose(out[starts[s] + i, h], want, rtol=0, atol=1e-12)


def test_one_new_token_per_sequence_is_decode():
    rng = np.random.default_rng(2)
    lens = [1, 5, 16, 17, 40]
    q, kc, vc, tables, lens_a, starts, _, _ = _problem(rng, lens, [1] * 5, 8, 2, 16)
    got = A.paged_prefill(q, kc, vc, tables, lens_a, starts, 0.25)
    want = A.paged_decode(q, kc, vc, tables, lens_a, 0.25)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_full_prompt_matches_torch_causal_sdpa(hq, hkv):
    rng = np.random.default_rng(3)
    lens = [7, 20, 1]
    q, kc, vc, tables, lens_a, starts, ks, vs = _problem(rng, lens, lens, hq, hkv, 8)
    scale = 0.4
    got = A.paged_prefill(q, kc, vc, tables, lens_a, starts, scale)
    g = hq // hkv
    for s, n in enumerate(lens):
        qt = torch.from_numpy(q[starts[s]: starts[s + 1]]).permute(1, 0, 2)           # [hq, n, d]
        kt = torch.from_numpy(ks[s]).repeat_interleave(g, dim=0)                        # [hq, n, d]
        vt = torch.from_numpy(vs[s]).repeat_interleave(g, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
        np.testing.assert_allclose(got[starts[s]: starts[s + 1]], ref.permute(1, 0, 2).numpy(),
                                   rtol=0, atol=1e-12)


def test_chunked_prefill_equals_one_prefill():
    """Prefilling a prompt in chunks (each chunk attending the cached earlier
    chunks) gives the rows of a single whole-prompt prefill."""
    rng = np.random.default_rng(4)
    n, hq, hkv, d = 23, 4, 2, 8
    q, kc, vc, tables, _, _, _, _ = _problem(rng, [n], [n], hq, hkv, d)
    whole = A.paged_prefill(q, kc, vc, tables, np.array([n]), np.array([0, n]), 0.5)
    done = 0
    for chunk in (5, 1, 9, 8):
        ctx = done + chunk
        part = A.paged_prefill(q[done:ctx], kc, vc, tables, np.array([ctx]), np.array([0, chunk]), 0.5)
        np.testing.assert_allclose(part, whole[done:ctx], rtol=0, atol=1e-12)
        done = ctx


def test_physical_placement_does_not_change_the_result():
    rng = np.random.default_rng(5)
    lens, qlens = [11, 30], [11, 7]
    q, kc, vc, tables, lens_a, starts, _, _ = _problem(rng, lens, qlens, 4, 2, 8)
    base = A.paged_prefill(q, kc, vc, tables, lens_a, starts, 0.5)
    perm = rng.permutation(kc.shape[0])              # move every block, rewrite the tables
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    assert np.array_equal(A.paged_prefill(q, kc2, vc2, tables2, lens_a, starts, 0.5), base)


def test_brute_force_tiny():
    rng = np.random.default_rng(6)
    lens, qlens = [3, 5], [2, 4]
    q, kc, vc, tables, lens_a, starts, ks, vs = _problem(rng, lens, qlens, 2, 1, 3, block_size=2)
    scale = 0.7
    got = A.paged_prefill(q, kc, vc, tables, lens_a, starts, scale)
    for s, (n, m) in enumerate(zip(lens, qlens)):
        for i in range(m):
            p = n - m + i
            for h in range(2):
                qv = [float(x) for x in q[starts[s] + i, h]]
                scores = [scale * sum(qv[c] * float(ks[s][0, j, c]) for c in range(3)) for j in range(p + 1)]
                mx = max(scores)
                e = [math.exp(x - mx) for x in scores]
                tot = sum(e)
                want = [sum(e[j] * float(vs[s][0, j, c]) for j in range(p + 1)) / tot for c in range(3)]
                np.testing.assert_allclose(got[starts[s] + i, h], want, rtol=0, atol=1e-12)


def test_sequence_subset_and_empty_queries():
    rng = np.random.default_rng(7)
    lens, qlens = [8, 12, 5], [3, 0, 5]
    q, kc, vc, tables, lens_a, starts, _, _ = _problem(rng, lens, qlens, 2, 2, 4)
    full = A.paged_prefill(q, kc, vc, tables, lens_a, starts, 0.5)
    assert full.shape[0] == 8
    sub = A.paged_prefill(q, kc, vc, tables, lens_a, starts, 0.5, seqs=[2, 0])
    np.testing.assert_array_equal(sub, np.concatenate([full[3:8], full[0:3]]))
