"""GPU parity of pa_decode_append (store the new token, then attend) against
the oracle.

Checked for every case: the caches after the call equal, bit for bit, the
oracle's append of each sequence's new rows at position context_lens[s] - 1;
the output matches the float64 oracle over the updated caches; and the output
and caches equal, bit for bit, those of pa_write_kv followed by pa_decode.
Cases cover the fast kernel storing the rows itself (MHA and GQA, head sizes
64 / 128 / 256, one to many partitions, the separate merge above 32
partitions, the new token at every kind of in-block offset), the paths with a
separate row-store kernel (fp32 caches, the generic path forced, a group of 5
query heads with head_dim 80, rows not 16-byte aligned on the fast and the
generic path), an invalid context length, and capture in a CUDA graph.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import assert_close_to_oracle, bits, needs_gpu
from oracle import attention as OA
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


def _new_rows(w, seed, misalign=False):
    g = syn.generator(seed, DEV)
    shape = (w.batch, w.n_kv_heads, w.head_dim)
    if not misalign:
        return syn.normal(shape, w.torch_dtype, DEV, g), syn.normal(shape, w.torch_dtype, DEV, g)
    # rows one element apart from 16-byte boundaries: a view of a wider buffer
    wide = (w.batch, w.n_kv_heads, w.head_dim + 1)
    k = syn.normal(wide, w.torch_dtype, DEV, g)[..., 1:]
    v = syn.normal(wide, w.torch_dtype, DEV, g)[..., 1:]
    return k, v


def check_append(w, seed, out_dtype=torch.float32, partition=512, misalign=False, path=0):
    inp = syn.decode_inputs(w, DEV)
    k_new, v_new = _new_rows(w, seed, misalign)
    maxc = int(w.lens.max())
    tables_np = inp.block_tables.cpu().numpy()
    want_k, want_v = OC.append_token(bits(k_new), bits(v_new), tables_np, w.lens, bits(inp.k_cache),
                                     bits(inp.v_cache))
    kc2, vc2 = inp.k_cache.clone(), inp.v_cache.clone()
    pk.set_decode_path(path)
    try:
        out = pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, inp.block_tables,
                               inp.context_lens, w.scale, maxc, partition, out_dtype=out_dtype)
        slots = torch.from_numpy(OC.last_token_slots(tables_np, w.lens, w.block_size).astype(np.int32)).to(DEV)
        pk.write_kv(k_new, v_new, slots, kc2, vc2)
        want = pk.decode(inp.q, kc2, vc2, inp.block_tables, inp.context_lens, w.scale, maxc, partition,
                         out_dtype=out_dtype)
        torch.cuda.synchronize()
    finally:
        pk.set_decode_path(0)
    assert pk.device_errors() == 0
    assert np.array_equal(bits(inp.k_cache), want_k) and np.array_equal(bits(inp.v_cache), want_v)
    ref = OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                          inp.context_lens.cpu(), w.scale)
    assert_close_to_oracle(out, ref, w.torch_dtype, "decode_append")
    assert torch.equal(out, want), "fused append differs from write_kv + decode"
    return out


# new token at offsets 0, 1, 7, 15 of its block, in the first and later
# partitions, one- and multi-partition sequences
RAGGED = [1, 2, 16, 17, 24, 511, 512, 513, 1000, 2048, 2049, 5000]


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (32, 8, 128, "bf16"),
    (32, 32, 128, "fp16"),
    (16, 16, 64, "bf16"),
    (32, 4, 256, "fp16"),
    (8, 1, 64, "bf16"),
    (128, 8, 128, "bf16"),
])
def test_fast_path_stores_rows_in_kernel(hq, hkv, d, dtype):
    w = syn.custom_workload(RAGGED, hq, hkv, d, dtype, seed=hq + hkv + d)
    check_append(w, seed=91)


def test_output_in_the_input_dtype():
    w = syn.custom_workload(RAGGED, 32, 8, 128, "bf16", seed=92)
    check_append(w, seed=93, out_dtype=torch.bfloat16)


def test_more_than_32_partitions_takes_the_separate_merge():
    w = syn.custom_workload([40 * 512 + 7, 300, 33 * 512], 32, 8, 128, "bf16", seed=94)
    check_append(w, seed=95)


def test_fp32_caches_store_rows_with_a_separate_kernel():
    w = syn.custom_workload([1, 17, 33, 64, 700], 4, 4, 64, "fp32", seed=96)
    check_append(w, seed=97)


def test_generic_path_rows_off_16_byte_boundaries():
    w = syn.custom_workload(RAGGED, 32, 8, 128, "fp16", seed=105)
    check_append(w, seed=106, misalign=True, path=1)


def test_generic_path_odd_group_and_head_size():
    # head_dim 80 takes the generic kernel and the separate row-store kernel,
    # with 5 query heads reading each KV head's new rows
    w = syn.custom_workload([1, 16, 17, 600, 1100], 10, 2, 80, "bf16", seed=107)
    check_append(w, seed=108)


def test_generic_path_forced():
    w = syn.custom_workload(RAGGED, 32, 8, 128, "fp16", seed=98)
    check_append(w, seed=99, path=1)


def test_rows_off_16_byte_boundaries_use_the_separate_kernel():
    w = syn.custom_workload(RAGGED, 32, 8, 128, "bf16", seed=100)
    check_append(w, seed=101, misalign=True)


def test_invalid_length_skips_that_sequence_only():
    w = syn.custom_workload([100, 600, 40], 32, 8, 128, "bf16", seed=102)
    inp = syn.decode_inputs(w, DEV)
    k_new, v_new = _new_rows(w, 103)
    lens = inp.context_lens.clone()
    lens[1] = 0                                              # invalid
    kc0 = bits(inp.k_cache)
    pk.device_errors()
    out = torch.full((3, 32, 128), float("nan"), device=DEV)
    pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, inp.block_tables, lens, w.scale, 600,
                     512, out=out)
    torch.cuda.synchronize()
    assert pk.device_errors() & pk._lib.PA_DEVERR_CONTEXT_LEN
    tables = inp.block_tables.cpu().numpy()
    good = [0, 2]
    want_k, _ = OC.append_token(bits(k_new)[good], bits(v_new)[good], tables[good], w.lens[good], kc0,
                                bits(inp.v_cache))
    assert np.array_equal(bits(inp.k_cache), want_k)        # sequence 1's block untouched
    assert torch.isnan(out[1]).all() and not torch.isnan(out[good]).any()


def test_decode_append_captured_in_a_cuda_graph():
    w = syn.custom_workload([100, 600, 1500, 33, 17], 32, 8, 128, "bf16", seed=104)
    inp = syn.decode_inputs(w, DEV)
    k_new, v_new = _new_rows(w, 105)
    maxc = int(w.lens.max())
    ws = torch.empty(pk.decode_workspace_size(w.batch, 32, 128, maxc, 512), dtype=torch.uint8, device=DEV)
    out = torch.empty(w.batch, 32, 128, dtype=torch.float32, device=DEV)
    kc_e, vc_e = inp.k_cache.clone(), inp.v_cache.clone()

    def step(kc, vc, o):
        pk.decode_append(inp.q, k_new, v_new, kc, vc, inp.block_tables, inp.context_lens, w.scale, maxc, 512,
                         out=o, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(inp.k_cache, inp.v_cache, out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(inp.k_cache, inp.v_cache, out)
    g = syn.generator(106, DEV)
    for rep in range(3):
        inp.q.copy_(syn.normal(inp.q.shape, torch.bfloat16, DEV, g))
        k_new.copy_(syn.normal(k_new.shape, torch.bfloat16, DEV, g))
        v_new.copy_(syn.normal(v_new.shape, torch.bfloat16, DEV, g))
        graph.replay()
        want = torch.empty_like(out)
        step(kc_e, vc_e, want)
        torch.cuda.synchronize()
        assert torch.equal(out, want), rep
        assert torch.equal(inp.k_cache, kc_e) and torch.equal(inp.v_cache, vc_e)
    assert pk.device_errors() == 0
    del graph


def test_empty_batch_is_a_no_op():
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device=DEV)
    kv = torch.empty(0, 2, 128, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    out = pk.decode_append(q, kv, kv, kc, vc, torch.empty(0, 4, dtype=torch.int32, device=DEV),
                           torch.empty(0, dtype=torch.int32, device=DEV), 0.1, 64, 512)
    torch.cuda.synchronize()
    assert out.shape == (0, 8, 128) and pk.device_errors() == 0
    assert not kc.any() and not vc.any()
