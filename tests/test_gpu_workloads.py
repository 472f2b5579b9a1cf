"""Full-size workloads in the launch configuration the benchmark times.

Outputs are checked on sampled sequences (the oracle recomputes each sampled
sequence from its own pages), and the sharing / copy-on-write workload is run
end to end through the C++ allocator, pa_copy_blocks, pa_write_kv and pa_decode
and compared with the oracle allocator + bitwise oracles.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import assert_close_to_oracle, bits, needs_gpu
from oracle import allocator as OAL
from oracle import attention as OA
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


def sampled_reference(inp, w, rows, k_cache=None, v_cache=None):
    """Oracle output for the listed sequences, from their own pages only
    (of ``inp``'s caches unless others are given)."""
    k_cache = inp.k_cache if k_cache is None else k_cache
    v_cache = inp.v_cache if v_cache is None else v_cache
    outs = []
    tables = inp.block_tables.cpu().numpy()
    for s in rows:
        nb = int(-(-w.lens[s] // w.block_size))
        ids = torch.from_numpy(tables[s, :nb].astype(np.int64)).to(DEV)
        kc = k_cache[ids].cpu()
        vc = v_cache[ids].cpu()
        outs.append(OA.paged_decode(inp.q[s:s + 1].cpu(), kc, vc, np.arange(nb)[None, :],
                                    np.array([w.lens[s]]), w.scale)[0])
    return np.stack(outs)


def pick_rows(w, k=6, seed=0):
    rng = np.random.default_rng(seed)
    order = np.argsort(w.lens)
    rows = {int(order[0]), int(order[-1])}
    rows.update(int(x) for x in rng.choice(w.batch, size=min(k, w.batch), replace=False))
    return sorted(rows)


@pytest.mark.parametrize("name", ["mha7b", "gqa", "long"])
def test_full_size_sampled(name):
    """pa_decode at full size; every sequence of the MHA and GQA workloads, a
    sample of the long-context one (checked in full in the test below)."""
    w = syn.workload(name)
    inp = syn.decode_inputs(w, DEV)
    maxc = int(w.lens.max())
    rows = pick_rows(w) if name == "long" else list(range(w.batch))
    ref = sampled_reference(inp, w, rows)
    out32 = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale,
                      maxc, w.partition_tokens, out_dtype=torch.float32)
    out16 = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale,
                      maxc, w.partition_tokens)
    assert pk.device_errors() == 0
    assert_close_to_oracle(out32[rows], ref, w.torch_dtype, f"{name} fp32 out")
    assert_close_to_oracle(out16[rows], ref, w.torch_dtype, f"{name} {w.dtype} out")
    # properties at every row: finite, and the 16-bit output is the rounding of the fp32 one
    assert torch.isfinite(out32).all()
    assert (out16.float() - out32).abs().max().item() <= 2 ** -7 * out32.abs().max().item() + 1e-6
    del inp
    torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mha7b", "gqa", "long"])
def test_full_size_bench_launch_every_sequence(name):
    """The benchmark's step at full size, as it launches it: pa_decode_append
    (store each sequence's new token, then attend) replayed from a CUDA graph,
    max_context above the longest sequence, a caller workspace, output in the
    input dtype (and, in the same graph, in fp32).  Caches are compared bit
    for bit with the oracle's slot placement of the new rows; every sequence's
    output with the float64 oracle over those caches."""
    w = syn.workload(name)
    inp = syn.decode_inputs(w, DEV)
    g = syn.generator(w.seed + 50, DEV)
    shape = (w.batch, w.n_kv_heads, w.head_dim)
    k_new = syn.normal(shape, w.torch_dtype, DEV, g)
    v_new = syn.normal(shape, w.torch_dtype, DEV, g)
    maxc = int(w.lens.max()) + 64
    ws = torch.empty(pk.decode_workspace_size(w.batch, w.n_q_heads, w.head_dim, maxc, w.partition_tokens),
                     dtype=torch.uint8, device=DEV)
    out16 = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=w.torch_dtype, device=DEV)
    out32 = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=DEV)

    # expected caches: the inputs with each new row at the oracle's slot
    slots = OC.last_token_slots(inp.block_tables.cpu().numpy(), w.lens, w.block_size)
    blk = torch.from_numpy(slots // w.block_size).to(DEV)
    off = torch.from_numpy(slots % w.block_size).to(DEV)
    want_k, want_v = inp.k_cache.clone(), inp.v_cache.clone()
    want_k[blk, :, off, :] = k_new
    want_v[blk, :, off, :] = v_new

    def step():
        for o in (out16, out32):   # the second call stores the same rows again
            pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens,
                             w.scale, maxc, w.partition_tokens, out=o, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    out16.zero_()
    out32.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    assert torch.equal(bits_view(inp.k_cache), bits_view(want_k))
    assert torch.equal(bits_view(inp.v_cache), bits_view(want_v))
    del graph, side
    rows = list(range(w.batch))
    ref = sampled_reference(inp, w, rows, want_k, want_v)
    assert_close_to_oracle(out32, ref, w.torch_dtype, f"{name} fp32 out")
    assert_close_to_oracle(out16, ref, w.torch_dtype, f"{name} {w.dtype} out")
    del inp, want_k, want_v
    torch.cuda.empty_cache()


def bits_view(t):
    return t.view({2: torch.int16, 4: torch.int32}[t.element_size()])


def sharing_workflow(n_prompts, prompt_len, n_samples, tails, heads, d, dtype, bitwise_oracle):
    """Drive the sharing workload through the product and the oracle allocator.

    Every append goes to both allocators and their slots / copy pairs must be
    identical.  K/V rows for each token are drawn once.  With
    ``bitwise_oracle`` the oracle caches are updated by the bitwise oracles and
    compared with the GPU caches; otherwise (full size, where copying the pool
    per step is too slow) each sample's gathered rows are compared with the
    exact rows written for it.
    """
    B = 16
    need = n_prompts * (-(-prompt_len // B)) + int(sum(-(-(prompt_len % B + int(t) + 1) // B) + 1
                                                       for t in tails.ravel()))
    NB = int(np.ceil(1.1 * need))
    order = np.random.default_rng(4).permutation(NB)
    pool = pk.BlockPool(NB, order)
    seqs = pk.SequenceTables(pool, B)
    opool = OAL.BlockPool(NB, order)
    oseqs = OAL.SequenceTables(opool, B)
    g = syn.generator(4, DEV)
    kc = torch.zeros(NB, heads, B, d, dtype=dtype, device=DEV)
    vc = torch.zeros_like(kc)
    ocache = [bits(kc), bits(vc)] if bitwise_oracle else None
    history = {}
    n_copies = 0

    def write(slots, oslots, pairs, opairs, sids):
        nonlocal n_copies
        n = len(oslots)
        k = syn.normal((n, heads, d), dtype, DEV, g)
        v = syn.normal((n, heads, d), dtype, DEV, g)
        if len(opairs):
            pk.copy_blocks([kc, vc], pairs.to(DEV))
            n_copies += len(opairs)
            if ocache is not None:
                ocache[:] = OC.copy_blocks(ocache, np.array(opairs))
        pk.write_kv(k, v, slots.to(DEV), kc, vc)
        if ocache is not None:
            ocache[:] = OC.write_kv(bits(k), bits(v), oslots, ocache[0], ocache[1])
        for i, sid in enumerate(sids):
            history.setdefault(sid, []).append((k[i], v[i]))

    groups = []
    for _ in range(n_prompts):
        p = seqs.add()
        assert oseqs.add() == p
        for t0 in range(0, prompt_len, 256):                 # prefill in chunks of 256 tokens
            n = min(256, prompt_len - t0)
            slots, pairs = seqs.append_n(p, n)
            oslots = [oseqs.append(p)[0] for _ in range(n)]
            assert slots == oslots and not pairs
            write(torch.tensor(slots, dtype=torch.int32), oslots, None, [], [p] * n)
        kids = [seqs.fork(p) for _ in range(n_samples - 1)]
        assert [oseqs.fork(p) for _ in range(n_samples - 1)] == kids
        for kid in kids:
            history[kid] = list(history[p])
        groups.append([p] + kids)
    samples = [s for grp in groups for s in grp]

    def step(sids):
        slots, pairs = seqs.append_arrays(sids)
        oslots, opairs = oseqs.append_many(sids)
        assert slots.tolist() == oslots and [tuple(x) for x in pairs.tolist()] == opairs
        write(slots, oslots, pairs, opairs, sids)

    flat_tails = tails.ravel()
    for r in range(int(tails.max())):                        # tails, in sample order each round
        active = [s for i, s in enumerate(samples) if flat_tails[i] > r]
        if active:
            step(active)
    step(samples)                                            # the measured decode step's write
    for s in samples:
        assert seqs.table(s) == oseqs.table(s)
    assert pool.refcounts() == opool.refcount and pool.free_list() == opool.free
    if ocache is not None:
        assert np.array_equal(bits(kc), ocache[0]) and np.array_equal(bits(vc), ocache[1])
    for s in samples:
        t = torch.tensor(seqs.table(s), dtype=torch.long, device=DEV)
        n = seqs.length(s)
        pos = torch.arange(n, device=DEV)
        got_k = kc[t[pos // B], :, pos % B]
        got_v = vc[t[pos // B], :, pos % B]
        want_k = torch.stack([kv[0] for kv in history[s]])
        want_v = torch.stack([kv[1] for kv in history[s]])
        assert np.array_equal(bits(got_k), bits(want_k)) and np.array_equal(bits(got_v), bits(want_v))
    return dict(seqs=seqs, samples=samples, kc=kc, vc=vc, n_copies=n_copies, groups=groups)


def test_sharing_workflow_small_bitexact():
    tails = np.random.default_rng(1).integers(0, 40, size=(3, 4), endpoint=True)
    r = sharing_workflow(3, 200, 4, tails, 6, 64, torch.float16, bitwise_oracle=True)
    assert r["n_copies"] == 3 * 3             # one copy per branching sample but the last writer
    seqs, samples = r["seqs"], r["samples"]
    max_blocks = max(len(seqs.table(s)) for s in samples)
    tables, lens = seqs.block_tables(samples, max_blocks)
    q = syn.normal((len(samples), 6, 64), torch.float16, DEV, syn.generator(7, DEV))
    out = pk.decode(q, r["kc"], r["vc"], tables.to(DEV), lens.to(DEV), 0.125, int(lens.max()), 512,
                    out_dtype=torch.float32)
    ref = OA.paged_decode(q.cpu(), r["kc"].cpu(), r["vc"].cpu(), tables.numpy(), lens.numpy(), 0.125)
    assert_close_to_oracle(out, ref, torch.float16, "sharing small")


@pytest.mark.slow
def test_sharing_workflow_full_size():
    """16 prompts x 1000 tokens, 8 samples, tails in [0, 256], 40 heads x 128, fp16."""
    tails = syn.cow_tails()
    r = sharing_workflow(16, 1000, 8, tails, 40, 128, torch.float16, bitwise_oracle=False)
    assert r["n_copies"] == 112
    seqs, samples = r["seqs"], r["samples"]
    for grp in r["groups"]:
        first = seqs.table(grp[0])
        for s in grp[1:]:
            assert seqs.table(s)[:62] == first[:62]       # 62 full prompt blocks stay shared
    max_blocks = max(len(seqs.table(s)) for s in samples)
    tables, lens = seqs.block_tables(samples, max_blocks)
    assert lens.tolist() == [1000 + int(t) + 1 for t in tails.ravel()]
    q = syn.normal((128, 40, 128), torch.float16, DEV, syn.generator(8, DEV))
    out = pk.decode(q, r["kc"], r["vc"], tables.to(DEV), lens.to(DEV), 128 ** -0.5, int(lens.max()), 512,
                    out_dtype=torch.float32)
    ref = OA.paged_decode(q.cpu(), r["kc"].cpu(), r["vc"].cpu(), tables.numpy(), lens.numpy(), 128 ** -0.5)
    assert_close_to_oracle(out, ref, torch.float16, "sharing full, every sequence")


def test_beam_search_caches_and_decode_match_the_oracle():
    """A beam-search process tree (fork on branching, free on pruning) with real
    K/V: every append writes its token through pa_write_kv after pa_copy_blocks
    of the step's copy-on-write pairs; the caches must equal the bitwise
    oracles' and decode over the surviving beams must match the oracle."""
    from test_beam_and_prefix import beam_trace

    ops, nb, B = beam_trace(11, width=4, steps=50, prompt=45, B=16, nb=300)
    H, D, dt = 4, 64, torch.bfloat16
    order = np.random.default_rng(2).permutation(nb)
    pool, opool = pk.BlockPool(nb, order), OAL.BlockPool(nb, order)
    seqs, oseqs = pk.SequenceTables(pool, B), OAL.SequenceTables(opool, B)
    kc = torch.zeros(nb, H, B, D, dtype=dt, device=DEV)
    vc = torch.zeros_like(kc)
    ocache = [bits(kc), bits(vc)]
    g = syn.generator(12, DEV)

    def write(slots, pairs):
        k = syn.normal((len(slots), H, D), dt, DEV, g)
        v = syn.normal((len(slots), H, D), dt, DEV, g)
        if pairs:
            pk.copy_blocks([kc, vc], torch.tensor(pairs, dtype=torch.int64, device=DEV))
            ocache[:] = OC.copy_blocks(ocache, np.array(pairs))
        pk.write_kv(k, v, torch.tensor(slots, dtype=torch.int32, device=DEV), kc, vc)
        ocache[:] = OC.write_kv(bits(k), bits(v), slots, ocache[0], ocache[1])

    for op in ops:
        if op[0] == "add":
            assert seqs.add() == oseqs.add()
        elif op[0] == "append_n":
            slots, pairs = seqs.append_n(op[1], op[2])
            oslots = [oseqs.append(op[1])[0] for _ in range(op[2])]
            assert slots == oslots and not pairs
            write(slots, [])
        elif op[0] == "append":
            slots, pairs = seqs.append(op[1])
            oslots, opairs = oseqs.append_many(op[1])
            assert slots == oslots and pairs == opairs
            write(slots, pairs)
        elif op[0] == "fork":
            assert seqs.fork(op[1]) == oseqs.fork(op[1]) == op[2]
        elif op[0] == "free":
            seqs.free(op[1])
            oseqs.free(op[1])
    assert np.array_equal(bits(kc), ocache[0]) and np.array_equal(bits(vc), ocache[1])
    live = seqs.live()
    tables, lens = seqs.block_tables(live, max(len(seqs.table(s)) for s in live))
    q = syn.normal((len(live), 8, D), dt, DEV, g)
    out = pk.decode(q, kc, vc, tables.to(DEV), lens.to(DEV), D ** -0.5, int(lens.max()), 32,
                    out_dtype=torch.float32)
    ref = OA.paged_decode(q.cpu(), kc.cpu(), vc.cpu(), tables.numpy(), lens.numpy(), D ** -0.5)
    assert_close_to_oracle(out, ref, dt, "beam search decode")


def test_decode_append_after_fork_and_copy_on_write():
    """A fork right before a step makes parent and child share a partial last
    block; the step's copy-on-write gives each its own block, and
    pa_decode_append then stores every new token and attends.  Caches and
    output equal pa_write_kv at the allocator's slots followed by pa_decode."""
    tails = np.random.default_rng(2).integers(0, 20, size=(2, 3), endpoint=True)
    r = sharing_workflow(2, 120, 3, tails, 4, 64, torch.bfloat16, bitwise_oracle=False)
    seqs, samples = r["seqs"], list(r["samples"])
    parent = next(s for s in samples if seqs.length(s) % 16)    # its last block is partial
    child = seqs.fork(parent)                       # shares every block of parent, the partial last one too
    ids = samples + [child]
    slots, pairs = seqs.append_arrays(ids)
    assert len(pairs) >= 1                          # the shared partial block was copied
    kc, vc = r["kc"], r["vc"]
    pk.copy_blocks([kc, vc], pairs.to(DEV))
    max_blocks = max(len(seqs.table(s)) for s in ids)
    tables, lens = seqs.block_tables(ids, max_blocks)
    g = syn.generator(11, DEV)
    k_new = syn.normal((len(ids), 4, 64), torch.bfloat16, DEV, g)
    v_new = syn.normal((len(ids), 4, 64), torch.bfloat16, DEV, g)
    q = syn.normal((len(ids), 4, 64), torch.bfloat16, DEV, g)
    kc2, vc2 = kc.clone(), vc.clone()
    maxc = int(lens.max())
    out = pk.decode_append(q, k_new, v_new, kc, vc, tables.to(DEV), lens.to(DEV), 0.125, maxc, 512,
                           out_dtype=torch.float32)
    pk.write_kv(k_new, v_new, slots.to(DEV), kc2, vc2)
    want = pk.decode(q, kc2, vc2, tables.to(DEV), lens.to(DEV), 0.125, maxc, 512, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    assert torch.equal(out, want)
    ref = OA.paged_decode(q.cpu(), kc.cpu(), vc.cpu(), tables.numpy(), lens.numpy(), 0.125)
    assert_close_to_oracle(out, ref, torch.bfloat16, "append after fork")
