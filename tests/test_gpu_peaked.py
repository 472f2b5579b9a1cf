"""GPU parity on peaked softmaxes whose running maximum moves far.

The N(0, 1) inputs of the other parity tests keep base-2 scores within about
+-6, so the online softmax hardly ever moves its running maximum after the
first keys, and the prefill kernel's lazy rescale of O in tensor memory (only
when a 64-key tile's maximum exceeds the running one by more than 8 in base 2)
never runs after the first tile.  Here q and K are built so that the scores
rise, fall, step, spike on the newest key, peak on one key in the middle,
step just under the threshold, spread widely or stay flat (tests/peaked.py),
with every score formed exactly by the kernels.  Each case is compared, element
by element, with the float64 oracle: the 2e-3 gate for 16-bit inputs (1e-5 for
fp32), and a precision bound derived from the arithmetic -- the two-term
split of P (the regression bound of the N(0, 1) tests) plus what an fp32
rounding of each scaled score (|score| < 2^10) can move the output.

Paths: pa_decode on the fast kernel (MHA; GQA groups 4, 8 and 16; head sizes
64, 128 and 256), on the generic kernel (16-bit and fp32), with one to ten
partitions merged in the kernel and with more than 32 merged by the separate
merge kernel; pa_decode_append; pa_prefill on the tensor-core kernel (groups 1,
4 and 16, head sizes 64, 128 and 256, unsplit and with the key split) and on
the generic kernel.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
import peaked as PK
from gpu_util import PRECISION, TOL, assert_close_to_oracle, bits, needs_gpu, ulp_of
from oracle import attention as OA
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"

LENS = [1, 2, 17, 64, 100, 513, 1000, 1500, 2100, 5000]
CAP_FP32 = 16.0     # fp32 inputs: the 1e-5 gate leaves room for this score range only


def bound(in_dtype, vals, scale, v_cache):
    s2max = PK.score_max(vals, scale)
    return PRECISION[in_dtype] + PK.rounding_bound(s2max, float(v_cache.float().abs().max()))


def check(out, ref, in_dtype, eps, what):
    """fp32 output: the gate and the derived bound; 16-bit output: within one
    ulp of the rounded oracle plus the derived bound."""
    got = out.detach().float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    if out.dtype == torch.float32:
        err = assert_close_to_oracle(out, ref, in_dtype, what)
        assert err <= eps, f"{what}: max abs error {err:.3e} > derived bound {eps:.3e}"
        return err
    rne = torch.from_numpy(ref).to(out.dtype).double().numpy()
    diff = np.abs(got - rne)
    lim = ulp_of(rne, out.dtype) * 1.0000001 + eps
    assert not (diff > lim).any(), f"{what}: {int((diff > lim).sum())} elements beyond 1 ulp + {eps:.2e}"
    return float(np.abs(got - ref).max())


def peaked_decode(w, seed, cap=PK.S2_CAP):
    inp = syn.decode_inputs(w, DEV)
    tables = inp.block_tables.cpu().numpy()
    vals = PK.column_values(w.lens, w.scale, w.torch_dtype, seed, tables.shape[1] * w.block_size, cap)
    PK.fill_cache(inp.k_cache, tables, w.lens, vals)
    PK.set_queries(inp.q, w.n_q_heads // w.n_kv_heads)
    return inp, vals


def oracle_decode(inp, w):
    return OA.paged_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                           inp.context_lens.cpu(), w.scale)


def run_decode(inp, w, out_dtype, partition, path):
    pk.set_decode_path(path)
    try:
        out = pk.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale,
                        int(w.lens.max()), partition, out_dtype=out_dtype)
        torch.cuda.synchronize()
    finally:
        pk.set_decode_path(0)
    assert pk.device_errors() == 0
    return out


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (8, 8, 128, "fp16"),      # fast MHA
    (8, 8, 128, "bf16"),
    (16, 16, 64, "bf16"),
    (8, 8, 256, "fp16"),
    (32, 8, 128, "bf16"),     # fast GQA, 4 heads per KV head
    (32, 8, 64, "fp16"),
    (16, 4, 256, "bf16"),
    (64, 8, 128, "bf16"),     # 8 heads per KV head
    (32, 2, 128, "bf16"),     # 16 heads per KV head
    (32, 2, 64, "fp16"),
])
def test_decode_fast_kernel_peaked(hq, hkv, d, dtype):
    w = syn.custom_workload(LENS, hq, hkv, d, dtype, seed=300 + hq + d)
    inp, vals = peaked_decode(w, seed=301)
    ref = oracle_decode(inp, w)
    eps = bound(w.torch_dtype, vals, w.scale, inp.v_cache)
    out = run_decode(inp, w, torch.float32, 512, 0)
    check(out, ref, w.torch_dtype, eps, f"decode {hq}/{hkv} d{d} {dtype}")
    out16 = run_decode(inp, w, None, 512, 0)
    check(out16, ref, w.torch_dtype, eps, f"decode {hq}/{hkv} d{d} {dtype}, {dtype} out")


@pytest.mark.parametrize("hq,hkv,d,dtype", [(32, 8, 128, "bf16"), (8, 8, 128, "fp16"), (24, 2, 96, "bf16")])
def test_decode_generic_kernel_peaked(hq, hkv, d, dtype):
    w = syn.custom_workload(LENS, hq, hkv, d, dtype, seed=310 + hq + d)
    inp, vals = peaked_decode(w, seed=311)
    ref = oracle_decode(inp, w)
    eps = bound(w.torch_dtype, vals, w.scale, inp.v_cache)
    out = run_decode(inp, w, torch.float32, 256, 1)
    check(out, ref, w.torch_dtype, eps, f"generic decode {hq}/{hkv} d{d} {dtype}")


def test_decode_fp32_peaked():
    """fp32 caches (generic kernel) against the 1e-5 gate, scores within +-16."""
    w = syn.custom_workload(LENS, 8, 4, 64, "fp32", seed=320)
    inp, vals = peaked_decode(w, seed=321, cap=CAP_FP32)
    ref = oracle_decode(inp, w)
    out = run_decode(inp, w, torch.float32, 512, 0)
    assert_close_to_oracle(out, ref, torch.float32, "fp32 decode, peaked")


@pytest.mark.parametrize("hq,hkv", [(8, 8), (32, 8), (32, 2)])
def test_decode_many_partitions_peaked(hq, hkv):
    """64-token partitions: 47 partitions for the longest sequence, so the
    separate merge kernel combines partition maxima hundreds apart."""
    w = syn.custom_workload([3000, 2048, 700, 65, 1], hq, hkv, 128, "bf16", seed=330 + hq)
    inp, vals = peaked_decode(w, seed=331)
    ref = oracle_decode(inp, w)
    eps = bound(w.torch_dtype, vals, w.scale, inp.v_cache)
    for part in (64, 512):
        out = run_decode(inp, w, torch.float32, part, 0)
        check(out, ref, w.torch_dtype, eps, f"decode {hq}/{hkv}, partition {part}")


@pytest.mark.parametrize("hq,hkv,d,dtype", [(32, 8, 128, "bf16"), (8, 8, 128, "fp16"), (32, 2, 128, "bf16")])
def test_decode_append_peaked(hq, hkv, d, dtype):
    """The appended row carries its position's pattern value (for the
    "last_key" column, the spike): caches bit-exact with the oracle's append,
    output against the oracle, and equal to pa_write_kv + pa_decode."""
    lens = [1, 2, 16, 17, 511, 512, 513, 1000, 2049, 5000]
    w = syn.custom_workload(lens, hq, hkv, d, dtype, seed=340 + hq)
    inp, vals = peaked_decode(w, seed=341)
    g = syn.generator(342, DEV)
    k_new = syn.normal((w.batch, hkv, d), w.torch_dtype, DEV, g)
    v_new = syn.normal((w.batch, hkv, d), w.torch_dtype, DEV, g)
    last = torch.from_numpy(w.lens - 1).to(DEV)
    P = vals.shape[2]
    k_new[:, :, :P] = vals.to(DEV)[torch.arange(w.batch, device=DEV), last].to(w.torch_dtype)[:, None, :]
    tables = inp.block_tables.cpu().numpy()
    want_k, want_v = OC.append_token(bits(k_new), bits(v_new), tables, w.lens, bits(inp.k_cache),
                                     bits(inp.v_cache))
    kc2, vc2 = inp.k_cache.clone(), inp.v_cache.clone()
    maxc = int(w.lens.max())
    out = pk.decode_append(inp.q, k_new, v_new, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens,
                           w.scale, maxc, 512, out_dtype=torch.float32)
    slots = torch.from_numpy(OC.last_token_slots(tables, w.lens, 16).astype(np.int32)).to(DEV)
    pk.write_kv(k_new, v_new, slots, kc2, vc2)
    want = pk.decode(inp.q, kc2, vc2, inp.block_tables, inp.context_lens, w.scale, maxc, 512,
                     out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    assert np.array_equal(bits(inp.k_cache), want_k) and np.array_equal(bits(inp.v_cache), want_v)
    ref = oracle_decode(inp, w)
    check(out, ref, w.torch_dtype, bound(w.torch_dtype, vals, w.scale, inp.v_cache), "decode_append, peaked")
    assert torch.equal(out, want), "fused append differs from write_kv + decode"


# ---------------------------------------------------------------- prefill --
PREFILL_CASES = [(1, 1), (64, 64), (65, 65), (300, 300), (700, 200), (1000, 37), (129, 129), (17, 5),
                 (450, 450)]


def peaked_prefill(w, seed):
    inp = syn.prefill_inputs(w, DEV)
    tables = inp.block_tables.cpu().numpy()
    vals = PK.column_values(w.lens, w.scale, w.torch_dtype, seed, tables.shape[1] * w.block_size)
    PK.fill_cache(inp.k_cache, tables, w.lens, vals)
    PK.set_queries(inp.q, w.n_q_heads // w.n_kv_heads)
    return inp, vals


def oracle_prefill(inp, w):
    return OA.paged_prefill(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.block_tables.cpu(),
                            inp.context_lens.cpu(), inp.query_start.cpu(), w.scale)


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (8, 8, 128, "bf16"),      # one query head per KV head
    (16, 16, 64, "fp16"),
    (32, 8, 128, "bf16"),     # 4 heads per KV head
    (16, 4, 64, "fp16"),
    (8, 2, 256, "bf16"),
    (32, 2, 128, "bf16"),     # 16 heads per KV head
    (32, 2, 64, "fp16"),
    (16, 16, 256, "fp16"),
])
def test_prefill_tensor_core_kernel_peaked(hq, hkv, d, dtype):
    w = syn.custom_prefill(*zip(*PREFILL_CASES), hq, hkv, d, dtype, seed=360 + hq + d)
    inp, vals = peaked_prefill(w, seed=351)
    ref = oracle_prefill(inp, w)
    eps = bound(w.torch_dtype, vals, w.scale, inp.v_cache)
    mq = int(w.qlens.max())
    out = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                     w.scale, mq, out_dtype=torch.float32)
    out16 = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, mq)
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    check(out, ref, w.torch_dtype, eps, f"prefill {hq}/{hkv} d{d} {dtype}")
    check(out16, ref, w.torch_dtype, eps, f"prefill {hq}/{hkv} d{d} {dtype}, {dtype} out")


@pytest.mark.parametrize("hq,hkv,d,dtype", [(32, 8, 128, "bf16"), (16, 16, 64, "fp16"), (16, 2, 256, "bf16")])
def test_prefill_key_split_peaked(hq, hkv, d, dtype):
    """Few rows over long contexts: each key partition keeps its own running
    maximum, and the merge combines partition maxima far apart."""
    w = syn.custom_prefill([20000, 5003, 3000], [64, 37, 1], hq, hkv, d, dtype, seed=370 + hq + d)
    inp, vals = peaked_prefill(w, seed=371)
    need = pk.prefill_workspace_size(int(w.qlens.sum()), hq, hkv, d, w.batch, 64,
                                     inp.block_tables.shape[1] * w.block_size)
    assert need > 0                                  # this launch splits its keys
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    split = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, 64, out_dtype=torch.float32, workspace=ws)
    whole = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                       w.scale, 64, out_dtype=torch.float32, workspace=torch.empty(0, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert pk.device_errors() == 0
    ref = oracle_prefill(inp, w)
    eps = bound(w.torch_dtype, vals, w.scale, inp.v_cache)
    check(split, ref, w.torch_dtype, eps, "split prefill, peaked")
    check(whole, ref, w.torch_dtype, eps, "unsplit prefill, peaked")


def test_prefill_generic_kernel_peaked():
    w = syn.custom_prefill(*zip(*PREFILL_CASES), 16, 4, 128, "fp16", seed=380)
    inp, vals = peaked_prefill(w, seed=381)
    pk.set_prefill_path(1)
    try:
        out = pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                         w.scale, int(w.qlens.max()), out_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        pk.set_prefill_path(0)
    assert pk.device_errors() == 0
    check(out, oracle_prefill(inp, w), w.torch_dtype, bound(w.torch_dtype, vals, w.scale, inp.v_cache),
          "generic prefill, peaked")
