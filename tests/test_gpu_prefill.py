"""GPU parity of pa_prefill against the float64 oracle.

Covers the tensor-core kernel (fp16 / bf16, head sizes 64, 128 and 256, query
heads per KV head 1, 2, 3, 4, 5, 6, 7, 8 and 16) and the CUDA-core kernel (fp32, forced generic
path), single- and multi-tile query chunks with ragged tails, cached prefixes
from none to several stages long, the new token alone (decode shape), empty
sequences, outputs in fp32 and in the input dtype, inconsistent lengths, a
sampled check of the full-size prefill workload and a full check of the
chunked-prefill workload.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import PRECISION, assert_close_to_oracle, assert_precise, needs_gpu
from oracle import attention as OA
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


def run_prefill(w, out_dtype=torch.float32, path=0, max_query_len=None):
    inp = syn.prefill_inputs(w, DEV)
    mq = int(w.qlens.max()) if max_query_len is None else max_query_len
    pk.set_prefill_path(path)
    try:
        out = torch.full(inp.q.shape, float("nan"), dtype=out_dtype, device=DEV)
        pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                   w.scale, mq, out=out)
        torch.cuda.synchronize()
    finally:
        pk.set_prefill_path(0)
    return inp, out


def oracle(inp, w, seqs=None):
    return OA.paged_prefill(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                            inp.context_lens.cpu(), inp.query_start.cpu(), w.scale, seqs=seqs)


# (context, new tokens): a lone new token, a whole prompt, chunks after short
# and long cached prefixes, tails of one and of 15 tokens past a block
CASES = [(1, 1), (16, 16), (17, 5), (100, 100), (700, 200), (1500, 37), (129, 129), (64, 1), (333, 300)]


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (32, 8, 128, "bf16"),
    (16, 16, 128, "fp16"),
    (8, 4, 64, "bf16"),
    (16, 2, 64, "fp16"),
    (8, 8, 64, "bf16"),
    (32, 8, 256, "bf16"),
    (16, 16, 256, "fp16"),
    (28, 4, 128, "bf16"),
    (48, 8, 64, "fp16"),
    (15, 3, 128, "bf16"),
    (128, 8, 128, "bf16"),
])
def test_tensor_core_kernel_matches_oracle(hq, hkv, d, dtype):
    lens, qlens = zip(*CASES)
    w = syn.custom_prefill(lens, qlens, hq, hkv, d, dtype, seed=hq * 7 + hkv + d)
    inp, out = run_prefill(w)
    assert pk.device_errors() == 0
    ref = oracle(inp, w)
    assert_close_to_oracle(out, ref, w.torch_dtype, "prefill")
    assert_precise(out, ref, w.torch_dtype, "prefill")


def test_output_in_the_input_dtype():
    lens, qlens = zip(*CASES)
    w = syn.custom_prefill(lens, qlens, 32, 8, 128, "bf16", seed=41)
    inp, out = run_prefill(w, out_dtype=torch.bfloat16)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), w.torch_dtype, "prefill bf16 out")


def test_generic_kernel_fp32_and_forced():
    w = syn.custom_prefill([17, 40, 5, 64], [17, 8, 5, 1], 4, 2, 64, "fp32", seed=42)
    inp, out = run_prefill(w)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.float32, "prefill fp32")
    w = syn.custom_prefill([300, 129, 16], [300, 64, 16], 32, 8, 128, "fp16", seed=43)
    inp, out = run_prefill(w, path=1)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.float16, "prefill generic")


def test_other_shapes_use_the_generic_kernel():
    # head_dim 96 and a group of 12 are outside the tensor-core kernel
    w = syn.custom_prefill([50, 20], [30, 20], 6, 2, 96, "bf16", seed=44)
    inp, out = run_prefill(w)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.bfloat16, "prefill d96 g3")
    w = syn.custom_prefill([50, 20], [30, 20], 24, 2, 64, "bf16", seed=45)
    inp, out = run_prefill(w)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.bfloat16, "prefill g12")


def test_empty_sequences_and_unowned_rows_are_not_written():
    w = syn.custom_prefill([40, 10, 90, 7], [0, 10, 0, 3], 8, 2, 128, "bf16", seed=45)
    inp = syn.prefill_inputs(w, DEV)
    extra = torch.zeros(2, 8, 128, dtype=torch.bfloat16, device=DEV)
    q = torch.cat([inp.q, extra])                   # two rows owned by no sequence
    out = torch.full(q.shape, float("nan"), device=DEV)
    pk.prefill(q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale, 10,
               out=out)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    ref = oracle(inp, w)
    assert_close_to_oracle(out[:13], ref, torch.bfloat16, "prefill with empty sequences")
    assert torch.isnan(out[13:]).all()


def test_inconsistent_lengths_are_flagged_and_skipped():
    w = syn.custom_prefill([40, 30, 20], [10, 5, 20], 8, 2, 128, "bf16", seed=46)
    inp = syn.prefill_inputs(w, DEV)
    lens = inp.context_lens.clone()
    lens[1] = 3                                     # fewer tokens than new tokens: invalid
    out = torch.full(inp.q.shape, float("nan"), device=DEV)
    pk.device_errors()
    pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, lens, inp.query_start, w.scale, 20, out=out)
    torch.cuda.synchronize()
    assert pk.device_errors() & pk._lib.PA_DEVERR_CONTEXT_LEN
    assert torch.isnan(out[10:15]).all()
    ref = oracle(inp, w, seqs=[0, 2])
    assert_close_to_oracle(torch.cat([out[:10], out[15:]]), ref, torch.bfloat16, "valid sequences")


def test_max_query_len_below_a_chunk_is_flagged():
    w = syn.custom_prefill([300], [300], 8, 8, 128, "bf16", seed=47)
    pk.device_errors()
    inp, out = run_prefill(w, max_query_len=200)   # tiles cover 256 rows of 300
    assert pk.device_errors() & pk._lib.PA_DEVERR_CONTEXT_LEN
    ref = oracle(inp, w)
    assert_close_to_oracle(out[:256], ref[:256], torch.bfloat16, "rows inside the tiles")


def test_chunked_prefill_matches_one_prefill():
    """The same prompt prefilled in two chunks or at once gives the same rows."""
    w = syn.custom_prefill([1000], [1000], 32, 8, 128, "bf16", seed=48)
    inp = syn.prefill_inputs(w, DEV)
    whole = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, 1000, out_dtype=torch.float32)
    a = 389
    first = pk.prefill(inp.q[:a], inp.k_cache, inp.v_cache, inp.block_tables,
                       torch.tensor([a], dtype=torch.int32, device=DEV),
                       torch.tensor([0, a], dtype=torch.int32, device=DEV), w.scale, a, out_dtype=torch.float32)
    second = pk.prefill(inp.q[a:], inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens,
                        torch.tensor([0, 1000 - a], dtype=torch.int32, device=DEV), w.scale, 1000 - a,
                        out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    both = torch.cat([first, second])
    assert (both - whole).abs().max().item() <= 2 * PRECISION[torch.bfloat16]


def test_full_size_prefill_workload_sampled():
    """The 32-request prefill workload: fp32 output and, as the benchmark
    launches it, output in the input dtype; sampled sequences against the
    oracle, every row finite."""
    w = syn.workload("prefill")
    inp, out = run_prefill(w)
    out16 = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, int(w.qlens.max()))
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    assert torch.isfinite(out).all() and torch.isfinite(out16.float()).all()
    starts = w.query_start()
    for s in (0, int(np.argmax(w.lens)), int(np.argmax(w.qlens)), w.batch - 1):
        ref = oracle(inp, w, seqs=[s])
        got = out[starts[s]: starts[s + 1]]
        assert_close_to_oracle(got, ref, w.torch_dtype, f"prefill workload sequence {s}")
        assert_precise(got, ref, w.torch_dtype, f"prefill workload sequence {s}")
        assert_close_to_oracle(out16[starts[s]: starts[s + 1]], ref, w.torch_dtype,
                               f"prefill workload sequence {s}, {w.dtype} out")


@pytest.mark.slow
def test_full_size_chunked_workload_every_sequence():
    """The chunked-prefill workload (4 requests, 64-256 new tokens after
    16K-32K cached prefixes) launched as the benchmark does (workspace
    allocated by the binding, so the keys are split): every sequence against
    the oracle, outputs in fp32 and in the input dtype."""
    w = syn.workload("chunked")
    inp = syn.prefill_inputs(w, DEV)
    mq = int(w.qlens.max())
    assert pk.prefill_workspace_size(int(w.qlens.sum()), w.n_q_heads, w.n_kv_heads, w.head_dim, w.batch, mq,
                                     inp.block_tables.shape[1] * w.block_size) > 0
    outs = [pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, mq, out_dtype=dt) for dt in (torch.float32, w.torch_dtype)]
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    ref = oracle(inp, w)
    assert_close_to_oracle(outs[0], ref, w.torch_dtype, "chunked workload, fp32 out")
    assert_precise(outs[0], ref, w.torch_dtype, "chunked workload, fp32 out")
    assert_close_to_oracle(outs[1], ref, w.torch_dtype, f"chunked workload, {w.dtype} out")


def test_prefill_captured_in_a_cuda_graph():
    """pa_write_kv of a chunk + pa_prefill captured once and replayed with new
    values written into the same buffers give the eager results bit for bit."""
    w = syn.custom_prefill([300, 77, 40], [300, 30, 1], 32, 8, 128, "bf16", seed=49)
    inp = syn.prefill_inputs(w, DEV)
    g = syn.generator(50, DEV)
    rows = int(w.qlens.sum())
    k_new = syn.normal((rows, 8, 128), torch.bfloat16, DEV, g)
    v_new = syn.normal((rows, 8, 128), torch.bfloat16, DEV, g)
    tables = inp.block_tables.cpu().numpy()
    slots = []
    for s, (n, q) in enumerate(zip(w.lens, w.qlens)):
        slots += [int(tables[s, p // 16]) * 16 + p % 16 for p in range(int(n - q), int(n))]
    slots = torch.tensor(slots, dtype=torch.int32, device=DEV)
    out = torch.empty(inp.q.shape, dtype=torch.float32, device=DEV)
    kc_e, vc_e = inp.k_cache.clone(), inp.v_cache.clone()

    def step(kc, vc, o):
        pk.write_kv(k_new, v_new, slots, kc, vc)
        pk.prefill(inp.q, kc, vc, inp.block_tables, inp.context_lens, inp.query_start, w.scale, 300, out=o)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(inp.k_cache, inp.v_cache, out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(inp.k_cache, inp.v_cache, out)
    for rep in range(2):
        for t in (inp.q, k_new, v_new):
            t.copy_(syn.normal(t.shape, torch.bfloat16, DEV, g))
        graph.replay()
        want = torch.empty_like(out)
        step(kc_e, vc_e, want)
        torch.cuda.synchronize()
        assert torch.equal(out, want), rep
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.bfloat16, "graph replay")
    del graph


def test_non_positive_scale_uses_the_generic_kernel():
    w = syn.custom_prefill([70, 20], [40, 20], 8, 2, 128, "bf16", seed=51)
    inp = syn.prefill_inputs(w, DEV)
    for scale in (-0.09, 0.0):
        out = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                         scale, 40, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert pk.device_errors() == 0
        ref = OA.paged_prefill(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                               inp.context_lens.cpu(), inp.query_start.cpu(), scale)
        assert_close_to_oracle(out, ref, torch.bfloat16, f"scale {scale}")


@pytest.mark.parametrize("hq,hkv,d,dtype", [(32, 8, 128, "bf16"), (16, 16, 64, "fp16"), (16, 2, 256, "bf16")])
def test_key_split_for_few_rows_over_long_contexts(hq, hkv, d, dtype):
    """Few new tokens after long cached prefixes: the launch splits the keys
    (its workspace is sized by pa_prefill_workspace_size) and merges the
    partitions; the result matches the oracle and the unsplit launch."""
    lens, qlens = [20000, 5003, 3000], [64, 37, 1]
    w = syn.custom_prefill(lens, qlens, hq, hkv, d, dtype, seed=hq + d + 60)
    inp = syn.prefill_inputs(w, DEV)
    max_tokens = inp.block_tables.shape[1] * 16
    need = pk.prefill_workspace_size(int(w.qlens.sum()), hq, hkv, d, w.batch, 64, max_tokens)
    assert need > 0                                  # this launch splits
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    split = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                       64, out_dtype=torch.float32, workspace=ws)
    whole = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                       64, out_dtype=torch.float32, workspace=torch.empty(0, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    ref = oracle(inp, w)
    assert_close_to_oracle(split, ref, w.torch_dtype, "split prefill")
    assert_precise(split, ref, w.torch_dtype, "split prefill")
    assert (split - whole).abs().max().item() <= 2 * PRECISION[w.torch_dtype]
    out16 = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, 64, workspace=ws)
    torch.cuda.synchronize()
    assert_close_to_oracle(out16, ref, w.torch_dtype, "split prefill, 16-bit out")


def test_key_split_when_the_grid_is_under_four_ctas_per_sm():
    """A (query tile, KV head) grid of about three CTAs per SM: the launch
    splits the keys (the threshold is four CTAs per SM), and the result
    matches the oracle and the unsplit launch."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    hq, hkv, d = 32, 2, 64                           # 16 query heads per KV head: 8 new tokens per tile
    tiles = (3 * sms + 4 * hkv - 1) // (4 * hkv)     # tiles per sequence for a grid of ~3 CTAs per SM
    mq = tiles * 8
    qlens = [mq, mq - 5, mq // 2, 9]
    lens = [2100 + q for q in qlens]
    w = syn.custom_prefill(lens, qlens, hq, hkv, d, "fp16", seed=68)
    inp = syn.prefill_inputs(w, DEV)
    max_tokens = inp.block_tables.shape[1] * 16
    assert 2 * sms < tiles * w.batch * hkv < 4 * sms
    need = pk.prefill_workspace_size(int(w.qlens.sum()), hq, hkv, d, w.batch, mq, max_tokens)
    assert need > 0                                  # this launch splits
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    split = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                       mq, out_dtype=torch.float32, workspace=ws)
    whole = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                       mq, out_dtype=torch.float32, workspace=torch.empty(0, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    ref = oracle(inp, w)
    assert_close_to_oracle(split, ref, w.torch_dtype, "split prefill, ~3 CTAs per SM")
    assert_precise(split, ref, w.torch_dtype, "split prefill, ~3 CTAs per SM")
    assert (split - whole).abs().max().item() <= 2 * PRECISION[w.torch_dtype]


def test_key_split_captured_in_a_cuda_graph():
    w = syn.custom_prefill([12000, 700], [32, 32], 32, 8, 128, "bf16", seed=66)
    inp = syn.prefill_inputs(w, DEV)
    need = pk.prefill_workspace_size(64, 32, 8, 128, 2, 32, inp.block_tables.shape[1] * 16)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out = torch.empty(inp.q.shape, dtype=torch.float32, device=DEV)

    def step(o):
        pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                   32, out=o, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(out)
    g = syn.generator(67, DEV)
    inp.q.copy_(syn.normal(inp.q.shape, torch.bfloat16, DEV, g))
    graph.replay()
    want = torch.empty_like(out)
    step(want)
    torch.cuda.synchronize()
    assert torch.equal(out, want)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out, oracle(inp, w), torch.bfloat16, "split prefill graph replay")
    del graph


def test_no_new_tokens_is_a_no_op():
    """Sequences with cached context but no new rows: nothing is launched or written."""
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device=DEV)
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device=DEV)
    tables = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device=DEV)
    lens = torch.tensor([20, 7], dtype=torch.int32, device=DEV)
    starts = torch.zeros(3, dtype=torch.int32, device=DEV)
    out = pk.prefill(q, kc, kc, tables, lens, starts, 0.1, 0)
    torch.cuda.synchronize()
    assert out.shape == (0, 8, 128) and pk.device_errors() == 0
