"""Pins for the float64 decode-attention oracle (CPU only).

The oracle is checked against things other than itself: a pure-Python scalar
brute force, closed forms, a hand-worked fixture, invariances the pages state
(physical placement is arbitrary; block size is a parameter; paging does not
change the attention result) and a library routine (torch's
scaled_dot_product_attention in float64).
"""

import math

import numpy as np
import pytest
import torch

from golden_io import read_kv
from oracle import attention as A

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- helpers ----

def _paged_from_contiguous(seqs_k, seqs_v, block_size, num_blocks, rng, fill=np.nan):
    """Scatter per-sequence contiguous [Hkv, n, d] arrays into a shuffled pool.

    Returns k_cache, v_cache [NB, Hkv, B, d], tables [batch, max_blocks], lens.
    Unused slots hold ``fill`` so that reading one poisons the result.
    """
    hkv, _, d = seqs_k[0].shape
    nbs = [-(-k.shape[1] // block_size) for k in seqs_k]
    num_blocks = max(num_blocks, sum(nbs) + 3)
    k_cache = np.full((num_blocks, hkv, block_size, d), fill)
    v_cache = np.full((num_blocks, hkv, block_size, d), fill)
    perm = rng.permutation(num_blocks)
    tables = np.full((len(seqs_k), max(nbs)), -1, np.int64)
    pos = 0
    for s, (K, V) in enumerate(zip(seqs_k, seqs_v)):
        n = K.shape[1]
        for i in range(nbs[s]):
            b = perm[pos]
            pos += 1
            tables[s, i] = b
            lo, hi = i * block_size, min(n, (i + 1) * block_size)
            k_cache[b, :, : hi - lo] = K[:, lo:hi]
            v_cache[b, :, : hi - lo] = V[:, lo:hi]
    lens = np.array([k.shape[1] for k in seqs_k], np.int64)
    return k_cache, v_cache, tables, lens


def _random_problem(rng, batch=3, hq=4, hkv=2, d=8, max_len=40):
    lens = rng.integers(1, max_len + 1, size=batch)
    ks = [rng.standard_normal((hkv, int(n), d)) for n in lens]
    vs = [rng.standard_normal((hkv, int(n), d)) for n in lens]
    q = rng.standard_normal((batch, hq, d))
    return q, ks, vs


def _brute_force(q, k_cache, v_cache, tables, lens, scale):
    """Scalar loops over nested Python lists: position -> (block, offset)."""
    q = q.tolist()
    kc = k_cache.tolist()
    vc = v_cache.tolist()
    block_size = len(kc[0][0])
    n_kv = len(kc[0])
    out = []
    for s in range(len(q)):
        n = int(lens[s])
        heads = []
        for h in range(len(q[s])):
            per_kv = len(q[s]) // n_kv
            hk = h // per_kv
            d = len(q[s][h])
            scores = []
            for pos in range(n):
                blk = int(tables[s][pos // block_size])
                off = pos % block_size
                dot = 0.0
                for e in range(d):
                    dot += q[s][h][e] * kc[blk][hk][off][e]
                scores.append(scale * dot)
            mx = max(scores)
            ws = [math.exp(x - mx) for x in scores]
            tot = sum(ws)
            row = []
            for e in range(d):
                acc = 0.0
                for pos in range(n):
                    blk = int(tables[s][pos // block_size])
                    acc += ws[pos] * vc[blk][hk][pos % block_size][e]
                row.append(acc / tot)
            heads.append(row)
        out.append(heads)
    return np.array(out)


# ------------------------------------------------------------------ pins ----

@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("block_size", [1, 2, 3, 16])
def test_brute_force_tiny(seed, block_size):
    rng = np.random.default_rng(seed)
    q, ks, vs = _random_problem(rng, batch=3, hq=4, hkv=2, d=3, max_len=9)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, block_size, 30, rng)
    got = A.paged_decode(q, kc, vc, tables, lens, 0.7)
    want = _brute_force(q, kc, vc, tables, lens, 0.7)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_golden_rational_weights():
    g = read_kv("decode_rational.txt")
    B, d, nb = g["block_size"], g["head_dim"], g["num_blocks"]
    kc = np.full((nb, 1, B, d), np.nan)
    vc = np.full((nb, 1, B, d), np.nan)
    keys = [[math.log(w), g["key_second"]] for w in g["weights"]]
    for pos in range(g["context_len"]):
        blk = g["block_table"][pos // B]
        kc[blk, 0, pos % B] = keys[pos]
        vc[blk, 0, pos % B] = g["v_rows"][pos]
    q = np.array([g["q"]], np.float64)
    out = A.paged_decode(q, kc, vc, np.array([g["block_table"]]), np.array([g["context_len"]]),
                         g["scale"])
    np.testing.assert_allclose(out[0], np.array(g["expected_out"]), rtol=0, atol=1e-12)


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(5)
    q, ks, vs = _random_problem(rng, batch=2, hq=2, hkv=2, d=16, max_len=1)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 8, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 0.25)
    for s in range(2):
        for h in range(2):
            assert np.array_equal(out[s, h], vs[s][h, 0])


def test_zero_query_and_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(6)
    q, ks, vs = _random_problem(rng, batch=2, hq=2, hkv=1, d=8, max_len=50)
    q[0] = 0.0                                 # zero query: uniform weights
    ks[1][:] = ks[1][:, :1, :]                 # equal keys: uniform weights
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 4, 40, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 1.0)
    for s in range(2):
        for h in range(2):
            np.testing.assert_allclose(out[s, h], vs[s][0].mean(axis=0), rtol=0, atol=1e-12)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(7)
    d, n = 8, 37
    K = rng.standard_normal((1, n, d))
    V = rng.standard_normal((1, n, d))
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    K[0, :, 0] = 0.0
    K[0, 23, 0] = 1000.0                       # score gap of 1000 -> weight 1 - e^-1000
    kc, vc, tables, lens = _paged_from_contiguous([K], [V], 16, 4, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 1.0)
    np.testing.assert_allclose(out[0, 0], V[0, 23], rtol=0, atol=1e-12)


def test_scale_enters_as_a_factor_on_scores():
    rng = np.random.default_rng(8)
    q, ks, vs = _random_problem(rng, batch=2, hq=2, hkv=2, d=8, max_len=30)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 4, 30, rng)
    a = A.paged_decode(q, kc, vc, tables, lens, 0.5)
    b = A.paged_decode(q * 0.5, kc, vc, tables, lens, 1.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    c = A.paged_decode(q, kc, vc, tables, lens, 2.0)
    assert np.abs(a - c).max() > 1e-3


def test_physical_placement_does_not_change_the_result():
    """Blocks live at arbitrary physical addresses; moving them changes nothing."""
    rng = np.random.default_rng(9)
    q, ks, vs = _random_problem(rng, batch=4, hq=4, hkv=2, d=8, max_len=70)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 40, rng)
    base = A.paged_decode(q, kc, vc, tables, lens, 0.3)
    perm = rng.permutation(kc.shape[0])        # physical block b moves to perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    moved = A.paged_decode(q, kc2, vc2, tables2, lens, 0.3)
    assert np.array_equal(base, moved)


def test_block_size_does_not_change_the_result():
    rng = np.random.default_rng(10)
    q, ks, vs = _random_problem(rng, batch=3, hq=4, hkv=4, d=8, max_len=100)
    outs = []
    for B in (1, 4, 8, 16, 32):
        kc, vc, tables, lens = _paged_from_contiguous(ks, vs, B, 120, np.random.default_rng(B))
        outs.append(A.paged_decode(q, kc, vc, tables, lens, 0.4))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=0, atol=1e-12)


def test_equals_unpaged_contiguous_attention():
    rng = np.random.default_rng(11)
    q, ks, vs = _random_problem(rng, batch=3, hq=6, hkv=3, d=16, max_len=90)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 30, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 0.25)
    for s in range(3):
        for h in range(6):
            hk = h // 2
            s_ = 0.25 * (ks[s][hk] @ q[s, h])
            w = np.exp(s_ - s_.max())
            ref = (w / w.sum()) @ vs[s][hk]
            np.testing.assert_allclose(out[s, h], ref, rtol=0, atol=1e-12)


def test_matches_torch_sdpa_in_float64():
    rng = np.random.default_rng(12)
    q, ks, vs = _random_problem(rng, batch=3, hq=8, hkv=2, d=32, max_len=200)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 50, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 1.0 / math.sqrt(32))
    for s in range(3):
        K = torch.from_numpy(ks[s]).repeat_interleave(4, dim=0)   # [Hq, n, d]
        V = torch.from_numpy(vs[s]).repeat_interleave(4, dim=0)
        Q = torch.from_numpy(q[s])[:, None, :]                      # [Hq, 1, d]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V)[:, 0, :]
        np.testing.assert_allclose(out[s], ref.numpy(), rtol=0, atol=1e-12)


def test_grouped_heads_read_their_own_kv_head():
    """Query head h reads KV head h // (Hq / Hkv): make each V head a constant."""
    rng = np.random.default_rng(13)
    hq, hkv, d, n = 8, 4, 4, 20
    K = rng.standard_normal((hkv, n, d))
    V = np.stack([np.full((n, d), float(hk)) for hk in range(hkv)])
    q = rng.standard_normal((1, hq, d))
    kc, vc, tables, lens = _paged_from_contiguous([K], [V], 16, 4, rng)
    out = A.paged_decode(q, kc, vc, tables, lens, 1.0)
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], np.full(d, float(h // 2)), rtol=0, atol=1e-12)


def test_unfilled_slots_and_unused_table_entries_are_not_read():
    rng = np.random.default_rng(14)
    q, ks, vs = _random_problem(rng, batch=2, hq=2, hkv=1, d=4, max_len=30)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 10, rng, fill=np.nan)
    out = A.paged_decode(q, kc, vc, tables, lens, 1.0)
    assert np.isfinite(out).all()


@pytest.mark.parametrize("chunk", [1, 5, 16, 512])
def test_split_context_merge_equals_unsplit(chunk):
    """Per-chunk (m, l, acc) states merged by log-sum-exp give the same output."""
    rng = np.random.default_rng(15)
    d, n = 16, 700
    K = rng.standard_normal((n, d)) * 3.0
    V = rng.standard_normal((n, d))
    q = rng.standard_normal(d)
    full = A.contiguous_attention(q, K, V, 0.5)
    states = [A.partial_state(q, K[i:i + chunk], V[i:i + chunk], 0.5) for i in range(0, n, chunk)]
    np.testing.assert_allclose(A.lse_merge(states), full, rtol=0, atol=1e-12)


def test_bf16_inputs_are_upcast_exactly():
    t = torch.randn(3, 1, 16, 8).to(torch.bfloat16)
    got = A.to_f64(t)
    assert got.dtype == np.float64
    assert np.array_equal(got, t.float().numpy().astype(np.float64))


def test_rows_subset_matches_full_batch():
    rng = np.random.default_rng(16)
    q, ks, vs = _random_problem(rng, batch=5, hq=4, hkv=2, d=8, max_len=40)
    kc, vc, tables, lens = _paged_from_contiguous(ks, vs, 16, 30, rng)
    full = A.paged_decode(q, kc, vc, tables, lens, 0.3)
    sub = A.paged_decode_rows(q, kc, vc, tables, lens, 0.3, [4, 1])
    assert np.array_equal(sub, full[[4, 1]])


def test_brute_force_helper_catches_a_dropped_term():
    """The brute force itself reacts to a missing token (guards the pin)."""
    rng = np.random.default_rng(17)
    K = rng.standard_normal((1, 5, 3))
    V = rng.standard_normal((1, 5, 3))
    q = rng.standard_normal((1, 1, 3))
    kc, vc, tables, lens = _paged_from_contiguous([K], [V], 2, 6, rng)
    a = _brute_force(q, kc, vc, tables, lens, 1.0)
    b = _brute_force(q, kc, vc, tables, lens - 1, 1.0)
    assert np.abs(a - b).max() > 1e-6
