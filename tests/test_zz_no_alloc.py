"""pa_decode_noalloc: decode for callers that may not allocate device memory.

Some callers cannot hand the library a scratch buffer -- an engine that gave
nearly all device memory to its KV block pool at start-up and allows no later
allocation, or a plain C host with no device allocator of its own.  For them
pa_decode_noalloc uses a scratch array built into the library.  This file
checks it through the C ABI against pa_decode (same tolerance as the other
decode tests), on two calls in a row with different batches so that the second
call runs over the first call's leftovers in the shared scratch; that a call
after the first leaves the device's free memory and torch's allocator
counters unchanged; that an empty batch (the set-up call an engine makes before
reserving its block pool) succeeds; and that an oversized batch or a malformed
q is refused before any launch.

It lives in its own file, named to be collected last.
"""

import ctypes

import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import assert_close_to_oracle, needs_gpu
from oracle import attention as OA
from paged_kv_cache_364_b200 import _lib
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


def _case(lens, hq, hkv, dtype, seed):
    w = syn.custom_workload(lens, hq, hkv, 128, dtype, seed=seed)
    return w, syn.decode_inputs(w, DEV)


def _noalloc_via_c_abi(inp, w, max_context, out):
    lib = pk.library()
    d = pk._desc
    rc = lib.pa_decode_noalloc(ctypes.byref(d(inp.q, "q")), ctypes.byref(d(inp.k_cache, "k")),
                               ctypes.byref(d(inp.v_cache, "v")), ctypes.byref(d(inp.block_tables, "t")),
                               ctypes.byref(d(inp.context_lens, "l")), float(w.scale), int(max_context), 512,
                               ctypes.byref(d(out, "out")),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.PA_OK, lib.pa_last_error().decode()
    return out


def test_noalloc_matches_pa_decode_on_two_calls_in_a_row():
    cases = [
        _case([1, 300, 1500, 2047, 5000, 16], 32, 8, "bf16", seed=71),            # GQA, up to 10 partitions
        _case([2048, 129, 700, 1999] * 4, 32, 32, "fp16", seed=72),                # MHA, other shapes
    ]
    for w, inp in cases:
        maxc = int(w.lens.max())
        want = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale, maxc,
                         512, out_dtype=torch.float32)
        got = torch.full_like(want, float("nan"))
        _noalloc_via_c_abi(inp, w, maxc, got)
        torch.cuda.synchronize()
        assert pk.device_errors() == 0
        ref = OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                              inp.context_lens.cpu(), w.scale)
        assert_close_to_oracle(got, ref, w.torch_dtype, "noalloc vs oracle")
        assert (got - want).abs().max().item() <= 2e-3
        assert torch.equal(got, want)          # same kernels, same order: identical bits


def test_noalloc_refuses_a_batch_larger_than_its_scratch():
    lib = pk.library()
    w = syn.workload("gqa", batch=64)
    inp = syn.decode_inputs(syn.custom_workload([16] * 4, 32, 8, 128, "bf16", seed=1), DEV)
    # a [64, 32, 128] query batch at 131072 tokens needs far more than 32 MiB of scratch
    q = torch.zeros(64, 32, 128, dtype=torch.bfloat16, device=DEV)
    tables = torch.zeros(64, 8192, dtype=torch.int32, device=DEV)
    lens = torch.ones(64, dtype=torch.int32, device=DEV)
    out = torch.zeros(64, 32, 128, dtype=torch.float32, device=DEV)
    assert pk.decode_workspace_size(64, 32, 128, 131072, 512) > pk.NOALLOC_SCRATCH_BYTES
    d = pk._desc
    rc = lib.pa_decode_noalloc(ctypes.byref(d(q, "q")), ctypes.byref(d(inp.k_cache, "k")),
                               ctypes.byref(d(inp.v_cache, "v")), ctypes.byref(d(tables, "t")),
                               ctypes.byref(d(lens, "l")), float(w.scale), 131072, 512, ctypes.byref(d(out, "o")),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.PA_ERR_ARG
    assert b"scratch" in lib.pa_last_error()
    assert torch.count_nonzero(out).item() == 0   # nothing was launched


def test_noalloc_call_allocates_no_device_memory():
    """After a first call (which may load the library's modules and with them
    the scratch array), further calls leave the device's free memory and
    torch's allocator counters exactly as they were."""
    w, inp = _case([1, 300, 1500, 2047, 5000, 16], 32, 8, "bf16", seed=73)
    maxc = int(w.lens.max())
    out = torch.empty(w.batch, 32, 128, dtype=torch.float32, device=DEV)
    _noalloc_via_c_abi(inp, w, maxc, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(2):
        _noalloc_via_c_abi(inp, w, maxc, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.memory_reserved() == reserved0
    assert pk.device_errors() == 0


def test_noalloc_empty_batch_and_malformed_q():
    lib = pk.library()
    w, inp = _case([16, 40], 32, 8, "bf16", seed=74)
    d = pk._desc
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    q0 = torch.empty(0, 32, 128, dtype=torch.bfloat16, device=DEV)
    out0 = torch.empty(0, 32, 128, dtype=torch.float32, device=DEV)
    t0 = torch.empty(0, 4, dtype=torch.int32, device=DEV)
    l0 = torch.empty(0, dtype=torch.int32, device=DEV)
    rc = lib.pa_decode_noalloc(ctypes.byref(d(q0, "q")), ctypes.byref(d(inp.k_cache, "k")),
                               ctypes.byref(d(inp.v_cache, "v")), ctypes.byref(d(t0, "t")), ctypes.byref(d(l0, "l")),
                               float(w.scale), 64, 512, ctypes.byref(d(out0, "o")), stream)
    assert rc == _lib.PA_OK, lib.pa_last_error().decode()
    bad = d(inp.q, "q")
    bad.shape[0] = -1                                  # a negative batch is refused up front
    out = torch.zeros(2, 32, 128, dtype=torch.float32, device=DEV)
    rc = lib.pa_decode_noalloc(ctypes.byref(bad), ctypes.byref(d(inp.k_cache, "k")),
                               ctypes.byref(d(inp.v_cache, "v")), ctypes.byref(d(inp.block_tables, "t")),
                               ctypes.byref(d(inp.context_lens, "l")), float(w.scale), 40, 512,
                               ctypes.byref(d(out, "o")), stream)
    assert rc == _lib.PA_ERR_ARG and b"batch" in lib.pa_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
