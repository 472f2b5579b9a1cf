"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before touching the GPU (CPU only: no kernel is launched here)."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_364_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    hdr = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", hdr)))


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = declared_functions()
    assert len(names) >= 30
    for name in names:
        assert hasattr(lib, name), f"{name} is not exported"
        assert name in _lib.SIGNATURES, f"{name} has no ctypes signature"


def test_version_and_strerror(lib):
    assert lib.pa_version().decode().count(".") == 2
    for code in (_lib.PA_OK, _lib.PA_ERR_ARG, _lib.PA_ERR_DTYPE, _lib.PA_ERR_OOM, _lib.PA_ERR_STATE,
                 _lib.PA_ERR_BOUNDS, _lib.PA_ERR_CUDA, _lib.PA_ERR_TIMEOUT):
        assert lib.pa_strerror(code)
    assert lib.pa_strerror(123) == b"unknown error"


def fake(shape, dtype, ptr=0x100000):
    """A descriptor with a fake device pointer: only argument checks may see it."""
    d = _lib.PaTensor()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    stride = 1
    strides = []
    for n in reversed(shape):
        strides.append(stride)
        stride *= n
    for i, (n, s) in enumerate(zip(shape, reversed(strides))):
        d.shape[i] = n
        d.stride[i] = s
    return d


def test_write_kv_rejects_bad_arguments(lib):
    k = fake([4, 2, 8], _lib.PA_F16)
    slots = fake([4], _lib.PA_I32)
    kc = fake([10, 2, 16, 8], _lib.PA_F16)
    bad_head = fake([10, 3, 16, 8], _lib.PA_F16)
    bad_dtype = fake([10, 2, 16, 8], _lib.PA_BF16)
    bad_slots = fake([5], _lib.PA_I32)
    slots64 = fake([4], _lib.PA_I64)
    by = ctypes.byref
    assert lib.pa_write_kv(by(k), by(k), by(slots), by(kc), by(bad_head), None) == _lib.PA_ERR_ARG
    assert lib.pa_write_kv(by(k), by(k), by(slots), by(kc), by(bad_dtype), None) == _lib.PA_ERR_DTYPE
    assert lib.pa_write_kv(by(k), by(k), by(bad_slots), by(kc), by(kc), None) == _lib.PA_ERR_ARG
    assert lib.pa_write_kv(by(k), by(k), by(slots64), by(kc), by(kc), None) == _lib.PA_ERR_ARG
    assert b"slot_mapping" in lib.pa_last_error()
    empty = fake([0, 2, 8], _lib.PA_F16)
    empty_slots = fake([0], _lib.PA_I32)
    assert lib.pa_write_kv(by(empty), by(empty), by(empty_slots), by(kc), by(kc), None) == _lib.PA_OK


def test_decode_rejects_bad_arguments(lib):
    by = ctypes.byref
    q = fake([2, 8, 64], _lib.PA_BF16)
    kc = fake([10, 2, 16, 64], _lib.PA_BF16)
    bt = fake([2, 4], _lib.PA_I32)
    cl = fake([2], _lib.PA_I32)
    out = fake([2, 8, 64], _lib.PA_F32)
    ws_need = lib.pa_decode_workspace_size(2, 8, 64, 64, 512)
    ws = fake([ws_need], _lib.PA_U8, ptr=0x200000)
    small_ws = fake([ws_need - 1], _lib.PA_U8, ptr=0x200000)
    unaligned_ws = fake([ws_need], _lib.PA_U8, ptr=0x200010)

    def call(q=q, k=kc, v=kc, bt=bt, cl=cl, ws=ws, out=out, part=512, maxc=64):
        return lib.pa_decode(by(q), by(k), by(v), by(bt), by(cl), 0.125, maxc, part, by(ws), by(out), None)

    assert call(k=fake([10, 3, 16, 64], _lib.PA_BF16), v=fake([10, 3, 16, 64], _lib.PA_BF16)) == _lib.PA_ERR_ARG
    assert call(v=fake([10, 2, 16, 64], _lib.PA_F16)) == _lib.PA_ERR_DTYPE
    assert call(out=fake([2, 8, 64], _lib.PA_F16)) == _lib.PA_ERR_DTYPE
    assert call(bt=fake([3, 4], _lib.PA_I32)) == _lib.PA_ERR_ARG
    assert call(cl=fake([2], _lib.PA_I64)) == _lib.PA_ERR_ARG
    assert call(part=24) == _lib.PA_ERR_ARG          # not a multiple of B = 16
    assert call(maxc=0) == _lib.PA_ERR_ARG
    assert call(ws=small_ws) == _lib.PA_ERR_ARG
    assert call(ws=unaligned_ws) == _lib.PA_ERR_ARG
    assert call(q=fake([2, 8, 1024], _lib.PA_BF16), k=fake([10, 2, 16, 1024], _lib.PA_BF16),
                v=fake([10, 2, 16, 1024], _lib.PA_BF16), out=fake([2, 8, 1024], _lib.PA_F32)) == _lib.PA_ERR_ARG
    empty_q = fake([0, 8, 64], _lib.PA_BF16)
    assert call(q=empty_q, bt=fake([0, 4], _lib.PA_I32), cl=fake([0], _lib.PA_I32),
                out=fake([0, 8, 64], _lib.PA_F32)) == _lib.PA_OK


def test_workspace_size_grows_with_partitions(lib):
    a = lib.pa_decode_workspace_size(4, 32, 128, 512, 512)
    b = lib.pa_decode_workspace_size(4, 32, 128, 513, 512)
    c = lib.pa_decode_workspace_size(4, 32, 128, 131072, 512)
    assert 0 < a < b < c
    assert c >= 4 * 32 * 256 * 128 * 4
    assert lib.pa_decode_workspace_size(4, 32, 128, 0, 512) == 0


def test_prefill_split_threshold_is_four_ctas_per_sm(lib):
    """pa_prefill splits the keys only when its (query tile, KV head) grid is
    under four CTAs per SM (148 SMs here: no GPU reports another count) and
    the keys allow at least two partitions of 1,024."""
    hq, hkv, d, batch, max_tokens = 32, 8, 128, 1, 32768   # 4 query heads per KV head: 32 new tokens per tile
    def size(tiles, mt=max_tokens):
        mq = tiles * 32
        return lib.pa_prefill_workspace_size(mq, hq, hkv, d, batch, mq, mt)
    assert size(73) > 0                       # 73 tiles x 8 KV heads = 584 CTAs < 4 x 148
    assert size(74) == 0                      # 592 CTAs: no split
    assert size(73, mt=2047) == 0             # under two partitions of 1,024 keys: no split
    # 584 CTAs -> 2 partitions: fp32 partial outputs plus (max, sum) per row and head
    rows = 73 * 32
    acc = 2 * rows * hq * d * 4
    assert size(73) == ((acc + 255) // 256) * 256 + 2 * rows * hq * 8


def test_copy_blocks_rejects_bad_arguments(lib):
    by = ctypes.byref
    caches = (_lib.PaTensor * 2)(fake([10, 2, 16, 8], _lib.PA_F16), fake([10, 2, 16, 8], _lib.PA_BF16))
    pairs = fake([3, 2], _lib.PA_I64)
    assert lib.pa_copy_blocks(caches, 2, by(pairs), None) == _lib.PA_ERR_ARG
    assert lib.pa_copy_blocks(caches, 1, by(fake([3, 2], _lib.PA_I32)), None) == _lib.PA_ERR_ARG
    assert lib.pa_copy_blocks(caches, 1, by(fake([0, 2], _lib.PA_I64)), None) == _lib.PA_OK


def test_options_roundtrip(lib):
    v = ctypes.c_int32(-1)
    assert lib.pa_get_option(_lib.PA_OPT_DECODE_PATH, ctypes.byref(v)) == 0 and v.value == 0
    assert lib.pa_set_option(_lib.PA_OPT_DECODE_PATH, 1) == 0
    assert lib.pa_get_option(_lib.PA_OPT_DECODE_PATH, ctypes.byref(v)) == 0 and v.value == 1
    assert lib.pa_set_option(_lib.PA_OPT_DECODE_PATH, 0) == 0
    assert lib.pa_set_option(_lib.PA_OPT_DECODE_PATH, 7) == _lib.PA_ERR_ARG
    assert lib.pa_set_option(99, 0) == _lib.PA_ERR_ARG


def test_checked_option_roundtrip(lib):
    v = ctypes.c_int32(-1)
    assert lib.pa_get_option(_lib.PA_OPT_CHECKED, ctypes.byref(v)) == 0 and v.value == 0   # off by default
    assert lib.pa_set_option(_lib.PA_OPT_CHECKED, 1) == 0
    assert lib.pa_get_option(_lib.PA_OPT_CHECKED, ctypes.byref(v)) == 0 and v.value == 1
    for bad in (2, -1):
        assert lib.pa_set_option(_lib.PA_OPT_CHECKED, bad) == _lib.PA_ERR_ARG
        assert b"PA_OPT_CHECKED" in lib.pa_last_error()
    assert lib.pa_get_option(_lib.PA_OPT_CHECKED, ctypes.byref(v)) == 0 and v.value == 1   # unchanged
    assert lib.pa_set_option(_lib.PA_OPT_CHECKED, 0) == 0
    assert lib.pa_get_option(_lib.PA_OPT_CHECKED, None) == _lib.PA_ERR_ARG
    # argument errors are still found on the host before any check runs
    assert lib.pa_set_option(_lib.PA_OPT_CHECKED, 1) == 0
    assert lib.pa_write_kv(None, None, None, None, None, None) == _lib.PA_ERR_ARG
    assert lib.pa_set_option(_lib.PA_OPT_CHECKED, 0) == 0


def test_product_refuses_cpu_tensors():
    import torch

    import paged_kv_cache_364_b200 as pk

    k = torch.zeros(1, 1, 8, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        pk.write_kv(k, k, torch.zeros(1, dtype=torch.int32), torch.zeros(2, 1, 16, 8, dtype=torch.float16),
                    torch.zeros(2, 1, 16, 8, dtype=torch.float16))


def test_read_probe_rejects_bad_arguments(lib):
    sink = ctypes.c_void_p(0x200000)
    buf = ctypes.c_void_p(0x100000)
    assert lib.pa_read_probe(buf, 64, None, None) == _lib.PA_ERR_ARG           # no sink
    assert lib.pa_read_probe(None, 64, sink, None) == _lib.PA_ERR_ARG          # no buffer
    assert lib.pa_read_probe(buf, 40, sink, None) == _lib.PA_ERR_ARG           # not whole 16-byte units
    assert lib.pa_read_probe(ctypes.c_void_p(0x100008), 64, sink, None) == _lib.PA_ERR_ARG   # misaligned
    assert lib.pa_read_probe(buf, 64, ctypes.c_void_p(0x200002), None) == _lib.PA_ERR_ARG  # misaligned sink
    assert lib.pa_read_probe(buf, 0, sink, None) == _lib.PA_OK                 # empty: nothing launched
