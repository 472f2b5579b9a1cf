"""Checked mode (PA_OPT_CHECKED) on the GPU.

A write into a block that another sequence still reads corrupts a shared
prefix without any fault ("Stop Wasting GPU Memory: A Deep Dive Into vLLM's
PagedAttention", "Copy-on-Write for Parallel Sampling": a shared block is
copied before a sequence writes into it).  In checked mode the cache
operations look for such inputs first.  For each entry point: an aliasing call
is refused with PA_ERR_BOUNDS, sets PA_DEVERR_ALIAS and writes nothing; a
valid call gives the same bits as with the mode off; inside a stream capture a
checked call is refused with PA_ERR_STATE.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import bits, needs_gpu
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import _lib
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


@pytest.fixture
def checked():
    pk.device_errors()
    pk.set_checked(True)
    yield
    pk.set_checked(False)


def _pool(nb=40, hkv=2, d=64, seed=0):
    g = syn.generator(seed, DEV)
    return (syn.normal((nb, hkv, 16, d), torch.bfloat16, DEV, g), syn.normal((nb, hkv, 16, d), torch.bfloat16, DEV, g),
            g)


def test_write_kv_duplicate_slots_are_refused(checked):
    kc, vc, g = _pool()
    k = syn.normal((6, 2, 64), torch.bfloat16, DEV, g)
    v = syn.normal((6, 2, 64), torch.bfloat16, DEV, g)
    before = bits(kc), bits(vc)
    for slots in ([3, 17, 40, 17, -1, 5], [1, 1, 2, 3, 4, 5], [0, 1, 2, 3, 4, 0]):
        with pytest.raises(_lib.PagedKVError) as e:
            pk.write_kv(k, v, torch.tensor(slots, dtype=torch.int32, device=DEV), kc, vc)
        assert e.value.code == _lib.PA_ERR_BOUNDS and "aliasing" in str(e.value)
        assert pk.device_errors() & _lib.PA_DEVERR_ALIAS
        assert np.array_equal(bits(kc), before[0]) and np.array_equal(bits(vc), before[1])


def test_write_kv_valid_slots_match_the_unchecked_write(checked):
    kc, vc, g = _pool(nb=300)
    T = 3000                                           # several chunks of the all-pairs check
    perm = np.random.default_rng(1).permutation(300 * 16)[:T].astype(np.int32)
    perm[::7] = -1                                     # skipped tokens may repeat
    k = syn.normal((T, 2, 64), torch.bfloat16, DEV, g)
    v = syn.normal((T, 2, 64), torch.bfloat16, DEV, g)
    want_k, want_v = OC.write_kv(bits(k), bits(v), perm, bits(kc), bits(vc))
    pk.write_kv(k, v, torch.from_numpy(perm).to(DEV), kc, vc)
    assert pk.device_errors() == 0
    assert np.array_equal(bits(kc), want_k) and np.array_equal(bits(vc), want_v)


def test_copy_blocks_overlapping_pairs_are_refused(checked):
    kc, vc, _ = _pool()
    before = bits(kc)
    for pairs in ([[1, 2], [3, 2]], [[1, 2], [2, 5]], [[4, 4]], [[7, 9], [9, 8], [10, 11]]):
        with pytest.raises(_lib.PagedKVError) as e:
            pk.copy_blocks([kc, vc], torch.tensor(pairs, dtype=torch.int64, device=DEV))
        assert e.value.code == _lib.PA_ERR_BOUNDS
        assert pk.device_errors() & _lib.PA_DEVERR_ALIAS
        assert np.array_equal(bits(kc), before)
    pairs = np.array([[1, 2], [3, 4], [1, 5], [6, 7]], np.int64)   # one source copied twice is fine
    want = OC.copy_blocks([bits(kc), bits(vc)], pairs)
    pk.copy_blocks([kc, vc], torch.from_numpy(pairs).to(DEV))
    assert pk.device_errors() == 0
    assert np.array_equal(bits(kc), want[0]) and np.array_equal(bits(vc), want[1])


def _append_case():
    w = syn.custom_workload([40, 100, 17, 600], 8, 2, 128, "bf16", seed=11)
    inp = syn.decode_inputs(w, DEV)
    g = syn.generator(12, DEV)
    k_new = syn.normal((w.batch, 2, 128), torch.bfloat16, DEV, g)
    v_new = syn.normal((w.batch, 2, 128), torch.bfloat16, DEV, g)
    return w, inp, k_new, v_new


def test_decode_append_into_a_block_another_sequence_reads_is_refused(checked):
    w, inp, k_new, v_new = _append_case()
    tables = inp.block_tables.clone()
    # sequence 1's newest block (position 99 -> logical block 6) is also
    # sequence 0's logical block 1: shared, and not copied before the write
    tables[1, 6] = tables[0, 1]
    # sequence 3 lists its newest block (logical 37) again at logical 2
    bad_self = inp.block_tables.clone()
    bad_self[3, 2] = bad_self[3, 37]
    for t, first in ((tables, 0), (bad_self, 3)):
        before = bits(inp.k_cache), bits(inp.v_cache)
        out = torch.full((w.batch, 8, 128), float("nan"), device=DEV)
        with pytest.raises(_lib.PagedKVError) as e:
            pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, t, inp.context_lens, w.scale, 600,
                             512, out=out)
        assert e.value.code == _lib.PA_ERR_BOUNDS and f"first at index {first}" in str(e.value)
        assert pk.device_errors() & _lib.PA_DEVERR_ALIAS
        assert np.array_equal(bits(inp.k_cache), before[0]) and np.array_equal(bits(inp.v_cache), before[1])
        assert torch.isnan(out).all()                  # nothing was launched


def test_decode_append_valid_batch_matches_the_unchecked_call(checked):
    w, inp, k_new, v_new = _append_case()
    kc2, vc2 = inp.k_cache.clone(), inp.v_cache.clone()
    got = pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens,
                           w.scale, 600, 512, out_dtype=torch.float32)
    assert pk.device_errors() == 0
    pk.set_checked(False)
    want = pk.decode_append(inp.q, k_new, v_new, kc2, vc2, inp.block_tables, inp.context_lens, w.scale, 600, 512,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.equal(inp.k_cache, kc2) and torch.equal(inp.v_cache, vc2)


def test_checked_call_inside_a_stream_capture_is_refused(checked):
    kc, vc, g = _pool()
    k = syn.normal((2, 2, 64), torch.bfloat16, DEV, g)
    slots = torch.tensor([1, 2], dtype=torch.int32, device=DEV)
    x = torch.zeros(4, device=DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    code = None
    with torch.cuda.graph(graph, stream=side):
        x.add_(1)
        try:
            pk.write_kv(k, k, slots, kc, vc)
        except _lib.PagedKVError as e:
            code = e.code
    assert code == _lib.PA_ERR_STATE
    graph.replay()
    torch.cuda.synchronize()
    assert x.sum().item() == 4.0
    del graph
