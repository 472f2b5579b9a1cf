"""GPU parity of pa_decode against the float64 oracle.

Covers both kernels (the TMA-staged fast kernel for fp16/bf16 with block size
16, and the generic CUDA-core kernel), MHA and GQA group sizes, head sizes 64,
128 and 256, single- and multi-partition contexts with ragged tails, outputs in
fp32 and in the input dtype, and the degenerate cases (one token, exactly one
block, exactly one partition, one token past it, empty batch).
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import assert_close_to_oracle, assert_precise, needs_gpu
from oracle import attention as OA
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


def run_case(w, out_dtype=None, partition_tokens=None, path=0, max_context=None):
    inp = syn.decode_inputs(w, DEV)
    part = partition_tokens or w.partition_tokens
    maxc = max_context or int(w.lens.max())
    pk.set_decode_path(path)
    try:
        out = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens,
                        w.scale, maxc, part, out_dtype=out_dtype)
        torch.cuda.synchronize()
    finally:
        pk.set_decode_path(0)
    assert pk.device_errors() == 0
    ref = OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                          inp.context_lens.cpu(), w.scale)
    return out, ref


def test_tiny_fp32_workload():
    w = syn.workload("tiny")
    out, ref = run_case(w)
    assert out.dtype == torch.float32
    assert_close_to_oracle(out, ref, torch.float32, "tiny")


EDGE_LENS = [1, 15, 16, 17, 63, 64, 65, 511, 512, 513, 1000, 1024, 1025, 2047]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("heads", [(8, 8), (8, 4), (16, 4), (16, 2), (32, 4)])
@pytest.mark.parametrize("head_dim", [64, 128, 256])
def test_fast_kernel_matches_oracle(dtype, heads, head_dim):
    hq, hkv = heads
    name = {torch.float16: "fp16", torch.bfloat16: "bf16"}[dtype]
    w = syn.custom_workload(EDGE_LENS, hq, hkv, head_dim, name, seed=hq * 1000 + head_dim)
    out, ref = run_case(w, out_dtype=torch.float32)
    assert_close_to_oracle(out, ref, dtype, f"{name} {heads} d{head_dim} fp32-out")
    assert_precise(out, ref, dtype, f"{name} {heads} d{head_dim} precision")
    out16, _ = run_case(w)
    assert_close_to_oracle(out16, ref, dtype, f"{name} {heads} d{head_dim} {name}-out")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("heads,head_dim", [((128, 8), 128), ((32, 2), 64), ((16, 1), 128)])
def test_fast_kernel_group_16(dtype, heads, head_dim):
    """16 query heads per KV head: two 8-head column tiles of the GQA MMAs."""
    hq, hkv = heads
    name = {torch.float16: "fp16", torch.bfloat16: "bf16"}[dtype]
    w = syn.custom_workload(EDGE_LENS, hq, hkv, head_dim, name, seed=hq * 7 + head_dim)
    out, ref = run_case(w, out_dtype=torch.float32)
    assert_close_to_oracle(out, ref, dtype, f"{name} {heads} d{head_dim} fp32-out")
    assert_precise(out, ref, dtype, f"{name} {heads} d{head_dim} precision")
    out16, _ = run_case(w)
    assert_close_to_oracle(out16, ref, dtype, f"{name} {heads} d{head_dim} {name}-out")
    gen, _ = run_case(w, out_dtype=torch.float32, path=1)
    assert (out - gen).abs().max().item() <= 2e-4


@pytest.mark.parametrize("partition_tokens", [64, 512])
def test_group_16_partitions(partition_tokens):
    w = syn.custom_workload([1, 17, 600, 9000, 40 * 512 + 3], 64, 4, 128, "bf16", seed=77)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=partition_tokens)
    assert_close_to_oracle(out, ref, torch.bfloat16, f"g16 partition {partition_tokens}")


@pytest.mark.parametrize("partition_tokens", [16, 48, 128, 512, 2048])
def test_partition_sizes(partition_tokens):
    w = syn.custom_workload([1, 16, 100, 777, 3001, 4096], 32, 8, 128, "bf16", seed=5)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=partition_tokens)
    assert_close_to_oracle(out, ref, torch.bfloat16, f"partition {partition_tokens}")


@pytest.mark.parametrize("dtype", ["fp16", "bf16", "fp32"])
@pytest.mark.parametrize("shape", [(4, 4, 64), (12, 4, 96), (48, 3, 40), (8, 8, 512), (20, 1, 128)])
def test_generic_kernel_matches_oracle(dtype, shape):
    hq, hkv, d = shape
    w = syn.custom_workload([1, 5, 16, 33, 700], hq, hkv, d, dtype, seed=d)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=256, path=1)
    assert_close_to_oracle(out, ref, syn.DTYPES[dtype], f"generic {dtype} {shape}")


@pytest.mark.parametrize("block_size", [1, 8, 32])
def test_generic_kernel_other_block_sizes(block_size):
    w = syn.custom_workload([1, 9, 40, 300], 8, 2, 64, "bf16", block_size=block_size, seed=block_size)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=4 * block_size)
    assert_close_to_oracle(out, ref, torch.bfloat16, f"block size {block_size}")


def test_fast_and_generic_agree_on_gqa():
    w = syn.custom_workload(EDGE_LENS, 32, 8, 128, "bf16", seed=9)
    fast, ref = run_case(w, out_dtype=torch.float32)
    gen, _ = run_case(w, out_dtype=torch.float32, path=1)
    assert_close_to_oracle(fast, ref, torch.bfloat16)
    assert_close_to_oracle(gen, ref, torch.bfloat16)
    assert (fast - gen).abs().max().item() < 2e-3


def test_non_finite_values_in_unfilled_slots_are_ignored():
    """Slots past a sequence's length may hold anything, including NaN / inf."""
    w = syn.custom_workload([3, 17, 530], 16, 4, 128, "bf16", seed=21)
    inp = syn.decode_inputs(w, DEV)
    tables = inp.block_tables.cpu().numpy()
    for s, n in enumerate(w.lens):
        last = tables[s, (n - 1) // 16]
        off = n % 16
        if off:
            inp.k_cache[last, :, off:] = float("nan")
            inp.v_cache[last, :, off:] = float("inf")
    out = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale,
                    int(w.lens.max()), 512, out_dtype=torch.float32)
    ref = OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                          inp.context_lens.cpu(), w.scale)
    assert_close_to_oracle(out, ref, torch.bfloat16, "poisoned tails")


def test_physical_placement_and_strided_q():
    """Same logical data at another placement, q as a strided view: same output."""
    w = syn.custom_workload([40, 600, 1500], 16, 4, 128, "fp16", seed=31)
    inp = syn.decode_inputs(w, DEV)
    out1 = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale,
                     1500, 512, out_dtype=torch.float32)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1)).to(DEV)
    k2 = torch.empty_like(inp.k_cache)
    v2 = torch.empty_like(inp.v_cache)
    k2[perm] = inp.k_cache
    v2[perm] = inp.v_cache
    t = inp.block_tables.long()
    t2 = torch.where(t >= 0, perm[t.clamp(min=0)], t).int()
    qpad = torch.zeros(w.batch, w.n_q_heads + 3, 128, dtype=inp.q.dtype, device=DEV)
    qpad[:, 1:1 + w.n_q_heads] = inp.q
    q2 = qpad[:, 1:1 + w.n_q_heads]
    out2 = pk.decode(q2, k2, v2, t2, inp.context_lens, w.scale, 1500, 512, out_dtype=torch.float32)
    assert torch.equal(out1, out2)


def test_empty_batch_is_a_no_op():
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device=DEV)
    out = pk.decode(q, kc, kc, torch.empty(0, 4, dtype=torch.int32, device=DEV),
                    torch.empty(0, dtype=torch.int32, device=DEV), 0.1, 64)
    assert out.shape == (0, 8, 128)


def test_invalid_lengths_and_block_ids_are_flagged_not_faulted():
    w = syn.custom_workload([20, 40, 300, 50], 8, 2, 128, "bf16", seed=41)
    inp = syn.decode_inputs(w, DEV)
    lens = inp.context_lens.clone()
    lens[1] = 0                                   # invalid length
    tables = inp.block_tables.clone()
    tables[2, 3] = w.num_blocks + 5               # invalid block id inside the context
    pk.device_errors()
    out = torch.full((w.batch, 8, 128), 7.0, device=DEV)
    pk.decode(inp.q, inp.k_cache, inp.v_cache, tables, lens, w.scale, 300, 512, out=out)
    bits_ = pk.device_errors()
    assert bits_ & pk._lib.PA_DEVERR_CONTEXT_LEN
    assert bits_ & pk._lib.PA_DEVERR_BLOCK_ID
    assert torch.all(out[1] == 7.0)               # invalid row left unwritten
    ref = OA.paged_decode(inp.q.cpu()[[0, 3]], inp.k_cache.cpu(), inp.v_cache.cpu(),
                          inp.block_tables.cpu()[[0, 3]], inp.context_lens.cpu()[[0, 3]], w.scale)
    assert_close_to_oracle(out[[0, 3]], ref, torch.bfloat16, "valid rows")
    for path in (1,):
        pk.set_decode_path(path)
        try:
            pk.decode(inp.q, inp.k_cache, inp.v_cache, tables, lens, w.scale, 300, 512, out=out)
        finally:
            pk.set_decode_path(0)
        b = pk.device_errors()
        assert b & pk._lib.PA_DEVERR_CONTEXT_LEN and b & pk._lib.PA_DEVERR_BLOCK_ID


def test_context_longer_than_max_context_is_flagged():
    w = syn.custom_workload([100, 200], 8, 8, 64, "fp16", seed=51)
    inp = syn.decode_inputs(w, DEV)
    pk.device_errors()
    pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale, 150, 64)
    assert pk.device_errors() & pk._lib.PA_DEVERR_CONTEXT_LEN


def test_bounded_wait_gives_up_and_reports():
    pk.device_errors()
    assert pk.selftest_bounded_wait(1000) & pk._lib.PA_DEVERR_WAIT_TIMEOUT
    assert pk.device_errors() == 0
    x = torch.ones(4, device=DEV)
    assert (x + 1).sum().item() == 8.0            # the context is still usable


def test_repeated_calls_reuse_workspace_without_clearing():
    w = syn.custom_workload([5, 900, 2000, 33], 32, 8, 128, "bf16", seed=61)
    inp = syn.decode_inputs(w, DEV)
    ws = torch.full((pk.decode_workspace_size(4, 32, 128, 2000),), 0xAB, dtype=torch.uint8, device=DEV)
    outs = [pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale, 2000,
                      512, out_dtype=torch.float32, workspace=ws) for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_step_captured_in_a_cuda_graph_matches_eager():
    """pa_write_kv + pa_decode captured once in a CUDA graph and replayed with
    new input values (same buffers) give the eager results."""
    w = syn.custom_workload([100, 600, 1500, 33], 32, 8, 128, "bf16", seed=81)
    inp = syn.decode_inputs(w, DEV)
    g = syn.generator(82, DEV)
    k_new = syn.normal((w.batch, 8, 128), torch.bfloat16, DEV, g)
    v_new = syn.normal((w.batch, 8, 128), torch.bfloat16, DEV, g)
    tables = inp.block_tables.cpu().numpy()
    slots = torch.tensor([int(tables[s, (n - 1) // 16]) * 16 + (n - 1) % 16 for s, n in enumerate(w.lens)],
                         dtype=torch.int32, device=DEV)
    maxc = int(w.lens.max())
    ws = torch.empty(pk.decode_workspace_size(w.batch, 32, 128, maxc, 512), dtype=torch.uint8, device=DEV)
    out = torch.empty(w.batch, 32, 128, dtype=torch.float32, device=DEV)
    kc_eager, vc_eager = inp.k_cache.clone(), inp.v_cache.clone()

    def step(kc, vc, o):
        pk.write_kv(k_new, v_new, slots, kc, vc)
        pk.decode(inp.q, kc, vc, inp.block_tables, inp.context_lens, w.scale, maxc, 512, out=o, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(inp.k_cache, inp.v_cache, out)          # warm outside capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(inp.k_cache, inp.v_cache, out)
    for rep in range(3):
        inp.q.copy_(syn.normal(inp.q.shape, torch.bfloat16, DEV, g))
        k_new.copy_(syn.normal(k_new.shape, torch.bfloat16, DEV, g))
        v_new.copy_(syn.normal(v_new.shape, torch.bfloat16, DEV, g))
        graph.replay()
        want = torch.empty_like(out)
        step(kc_eager, vc_eager, want)
        torch.cuda.synchronize()
        assert torch.equal(out, want), rep
        assert torch.equal(inp.k_cache, kc_eager) and torch.equal(inp.v_cache, vc_eager)
    assert pk.device_errors() == 0
    ref = OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                          inp.context_lens.cpu(), w.scale)
    assert_close_to_oracle(out, ref, torch.bfloat16, "graph replay")
    del graph


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(6, 2, 50), (4, 4, 7)])
def test_generic_kernel_head_dims_off_four_through_the_merge(dtype, shape):
    """Head sizes that are not a multiple of 4 (the merge kernel's per-element
    path), many partitions per sequence (64-token partitions), merged by the
    separate merge kernel."""
    hq, hkv, d = shape
    w = syn.custom_workload([1, 33, 700, 1500], hq, hkv, d, dtype, seed=d + 500)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=64, path=1)
    assert_close_to_oracle(out, ref, syn.DTYPES[dtype], f"generic {dtype} {shape} off-4 head_dim")


def test_more_sequences_than_plan_threads():
    """1,500 sequences: the plan kernel's threads take two sequences each
    (its other path writes each thread's records itself), with single- and
    multi-partition sequences mixed; every sequence against the oracle."""
    rng = np.random.default_rng(404)
    lens = rng.integers(1, 200, size=1500)
    lens[::97] = rng.integers(600, 1800, size=len(lens[::97]))
    w = syn.custom_workload(lens, 8, 2, 64, "bf16", seed=405)
    out, ref = run_case(w, out_dtype=torch.float32)
    assert_close_to_oracle(out, ref, torch.bfloat16, "1,500 sequences")


@pytest.mark.parametrize("lens_kind", ["gqa", "mixed", "long"])
def test_plan_lists_every_partition_once_in_size_order(lens_kind):
    """The plan kernel's work list, read back from the workspace (header: item
    count; then one int4 record {sequence, partition, length, pages} per
    item): every (sequence, partition) exactly once with its length and page
    count, the full partitions first, then the rest by non-increasing size."""
    rng = np.random.default_rng({"gqa": 1, "mixed": 2, "long": 3}[lens_kind])
    if lens_kind == "gqa":
        lens = syn.workload("gqa").lens
    elif lens_kind == "mixed":
        lens = rng.integers(1, 3000, size=300)
    else:
        lens = rng.integers(20000, 60000, size=6)
    w = syn.custom_workload(lens, 8, 2, 128, "bf16", seed=7)
    inp = syn.decode_inputs(w, DEV)
    maxc = int(w.lens.max())
    ws = torch.zeros(pk.decode_workspace_size(w.batch, 8, 128, maxc, 512), dtype=torch.uint8, device=DEV)
    pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale, maxc, 512, workspace=ws)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    raw = ws.cpu().numpy()
    n_items = int(raw[:4].view(np.int32)[0])
    recs = raw[256:256 + 16 * n_items].view(np.int32).reshape(n_items, 4)
    nb = -(-w.lens // 16)
    want = set()
    for s, b in enumerate(nb):
        for q in range(-(-int(b) // 32)):
            want.add((s, q))
    got = [(int(r[0]), int(r[1])) for r in recs]
    assert len(got) == len(set(got)) and set(got) == want
    sizes = []
    for s, q, n, pages in recs:
        assert n == w.lens[s]
        assert pages == min(32, int(nb[s]) - 32 * q)
        sizes.append(int(pages))
    n_full = sum(1 for s, q, n, pages in recs if pages == 32)
    assert all(p == 32 for p in sizes[:n_full])
    rest = sizes[n_full:]
    assert all(a >= b for a, b in zip(rest, rest[1:]))


@pytest.mark.parametrize("heads,head_dim", [((12, 4), 128), ((15, 3), 64), ((12, 2), 128), ((14, 2), 64)])
@pytest.mark.parametrize("partition_tokens", [512, 64])
def test_fast_kernel_groups_3_5_6_7(heads, head_dim, partition_tokens):
    """Groups of 3, 5, 6 and 7 query heads per KV head on the tensor-core
    path; the in-kernel merge takes heads four at a time, so these end with a
    partial chunk.  64-token partitions give up to 32 partitions per row."""
    hq, hkv = heads
    lens = EDGE_LENS if partition_tokens == 512 else [1, 63, 64, 65, 700, 2047]
    w = syn.custom_workload(lens, hq, hkv, head_dim, "bf16", seed=hq * 11 + head_dim + partition_tokens)
    out, ref = run_case(w, out_dtype=torch.float32, partition_tokens=partition_tokens)
    assert_close_to_oracle(out, ref, torch.bfloat16, f"{heads} d{head_dim} partition {partition_tokens}")
    assert_precise(out, ref, torch.bfloat16, f"{heads} d{head_dim} partition {partition_tokens}")
