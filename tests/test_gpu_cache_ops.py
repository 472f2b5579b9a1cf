"""GPU parity of pa_write_kv and pa_copy_blocks against the bitwise oracle."""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import bits, needs_gpu
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda"


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("shape", [(37, 4, 64), (256, 8, 128), (5, 3, 40), (1, 1, 8)])
def test_write_kv_bitwise(dtype, shape):
    T, H, D = shape
    B, NB = 16, 3 * T // 16 + 8
    g = syn.generator(11, DEV)
    kc = syn.normal((NB, H, B, D), dtype, DEV, g)
    vc = syn.normal((NB, H, B, D), dtype, DEV, g)
    k = syn.normal((T, H, D), dtype, DEV, g)
    v = syn.normal((T, H, D), dtype, DEV, g)
    rng = np.random.default_rng(T)
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int32)
    slots[rng.random(T) < 0.2] = -1
    want_k, want_v = OC.write_kv(bits(k), bits(v), slots, bits(kc), bits(vc))
    pk.write_kv(k, v, torch.from_numpy(slots).to(DEV), kc, vc)
    assert np.array_equal(bits(kc), want_k)
    assert np.array_equal(bits(vc), want_v)
    assert pk.device_errors() == 0


def test_write_kv_strided_inputs():
    T, H, D, B, NB = 33, 4, 128, 16, 20
    g = syn.generator(12, DEV)
    kc = syn.normal((NB, H, B, D), torch.bfloat16, DEV, g)
    vc = kc.clone()
    kv = syn.normal((T, 2, H, D), torch.bfloat16, DEV, g)       # fused k|v projection output
    k, v = kv[:, 0], kv[:, 1]
    slots = np.random.default_rng(3).choice(NB * B, size=T, replace=False).astype(np.int32)
    want_k, want_v = OC.write_kv(bits(k), bits(v), slots, bits(kc), bits(vc))
    pk.write_kv(k, v, torch.from_numpy(slots).to(DEV), kc, vc)
    assert np.array_equal(bits(kc), want_k) and np.array_equal(bits(vc), want_v)


def test_write_kv_out_of_pool_slot_is_skipped_and_flagged():
    T, H, D, B, NB = 4, 2, 64, 16, 4
    g = syn.generator(13, DEV)
    kc = syn.normal((NB, H, B, D), torch.float16, DEV, g)
    vc = kc.clone()
    k = syn.normal((T, H, D), torch.float16, DEV, g)
    slots = np.array([3, NB * B, 7, -5], np.int32)     # two invalid slots
    before_k = bits(kc)
    pk.device_errors()
    pk.write_kv(k, k, torch.from_numpy(slots).to(DEV), kc, vc)
    assert pk.device_errors() & pk._lib.PA_DEVERR_SLOT
    want_k, _ = OC.write_kv(bits(k)[[0, 2]], bits(k)[[0, 2]], [3, 7], before_k, before_k)
    assert np.array_equal(bits(kc), want_k)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n_caches", [1, 2, 80])
def test_copy_blocks_bitwise(dtype, n_caches):
    NB, H, B, D = 40, 3, 16, 64
    g = syn.generator(14, DEV)
    caches = [syn.normal((NB, H, B, D), dtype, DEV, g) for _ in range(n_caches)]
    rng = np.random.default_rng(n_caches)
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:7], perm[7:14]], axis=1).astype(np.int64)
    want = OC.copy_blocks([bits(c) for c in caches], pairs)
    pk.copy_blocks(caches, torch.from_numpy(pairs).to(DEV))
    for c, w in zip(caches, want):
        assert np.array_equal(bits(c), w)
    assert pk.device_errors() == 0


def test_copy_blocks_odd_block_bytes_and_bad_pair():
    NB = 9
    g = syn.generator(15, DEV)
    c = syn.normal((NB, 3, 5), torch.float16, DEV, g)   # 30-byte blocks: 2-byte vectors
    pairs = np.array([[0, 4], [2, NB + 3], [1, 6]], np.int64)
    want = OC.copy_blocks([bits(c)], pairs[[0, 2]])[0]
    pk.device_errors()
    pk.copy_blocks([c], torch.from_numpy(pairs).to(DEV))
    assert pk.device_errors() & pk._lib.PA_DEVERR_COPY_PAIR
    assert np.array_equal(bits(c), want)


def test_copy_blocks_sharing_workload_size():
    """112 pairs x (K, V) of 40 heads x 16 x 128 fp16: the copy-on-write batch."""
    NB, H, B, D = 16 * 63 + 112 + 64, 40, 16, 128
    g = syn.generator(16, DEV)
    kc = syn.normal((NB, H, B, D), torch.float16, DEV, g)
    vc = syn.normal((NB, H, B, D), torch.float16, DEV, g)
    rng = np.random.default_rng(4)
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:112], perm[112:224]], axis=1).astype(np.int64)
    want = OC.copy_blocks([bits(kc)[:, :], bits(vc)], pairs)
    pk.copy_blocks([kc, vc], torch.from_numpy(pairs).to(DEV))
    assert np.array_equal(bits(kc), want[0]) and np.array_equal(bits(vc), want[1])
