"""B200-native paged KV cache: slot writes, paged decode attention, block copies
and the block allocator, behind the C ABI of ``libpagedkv.so``.

This module only marshals arguments: torch tensors become ``pa_tensor``
descriptors and the current CUDA stream is passed through.  Every step of the
path runs in the library's CUDA kernels or its C++ allocator; there is no
Python or CPU implementation to fall back on, and calls on CPU tensors raise.

    write_kv(k, v, slot_mapping, k_cache, v_cache)
    decode(q, k_cache, v_cache, block_tables, context_lens, scale, max_context, ...)
    copy_blocks(caches, src_dst_pairs)
    BlockPool / SequenceTables    host allocator (free pool, refcounts, tables)
"""

from __future__ import annotations

import ctypes
import struct

import torch

from . import _lib
from ._lib import AllocatorStateError, OutOfBlocks, PagedKVError  # noqa: F401

__all__ = [
    "write_kv", "decode", "decode_append", "decode_noalloc", "decode_workspace_size", "prefill",
    "prefill_workspace_size",
    "set_prefill_path", "get_prefill_path", "copy_blocks", "device_errors",
    "set_decode_path", "get_decode_path", "selftest_bounded_wait", "profile_enable", "profile_take", "BlockPool", "SequenceTables", "PagedKVError",
    "OutOfBlocks", "AllocatorStateError", "library", "version", "launch_count",
]

_DTYPES = {
    torch.float32: _lib.PA_F32,
    torch.float16: _lib.PA_F16,
    torch.bfloat16: _lib.PA_BF16,
    torch.int32: _lib.PA_I32,
    torch.int64: _lib.PA_I64,
    torch.uint8: _lib.PA_U8,
}


def library():
    """The loaded ctypes library (built in-tree on first use)."""
    return _lib.load()


def version() -> str:
    return library().pa_version().decode()


def launch_count() -> int:
    """CUDA kernels this library has enqueued since it was loaded."""
    n = ctypes.c_uint64(0)
    _lib.check(library().pa_launch_count(ctypes.byref(n)), "pa_launch_count")
    return int(n.value)


def _desc(t: torch.Tensor, name: str) -> _lib.PaTensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in _DTYPES:
        raise TypeError(f"{name}: unsupported dtype {t.dtype}")
    if t.dim() > _lib.MAX_DIMS:
        raise ValueError(f"{name}: rank above {_lib.MAX_DIMS}")
    d = _lib.PaTensor()
    d.data = t.data_ptr() if t.numel() else None
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i, (n, s) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = n
        d.stride[i] = s
    return d


def _device_tensors(*named):
    dev = None
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    return dev


def _stream(dev, stream):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream)


def write_kv(k, v, slot_mapping, k_cache, v_cache, stream=None):
    """Store token rows k[t], v[t] into slot slot_mapping[t] (-1 skips)."""
    dev = _device_tensors(("k", k), ("v", v), ("slot_mapping", slot_mapping),
                          ("k_cache", k_cache), ("v_cache", v_cache))
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_write_kv(ctypes.byref(_desc(k, "k")), ctypes.byref(_desc(v, "v")),
                             ctypes.byref(_desc(slot_mapping, "slot_mapping")),
                             ctypes.byref(_desc(k_cache, "k_cache")),
                             ctypes.byref(_desc(v_cache, "v_cache")), _stream(dev, stream))
    _lib.check(rc, "pa_write_kv")


def decode_workspace_size(batch, num_q_heads, head_dim, max_context, partition_tokens=512) -> int:
    n = library().pa_decode_workspace_size(batch, num_q_heads, head_dim, max_context, partition_tokens)
    if n == 0 and batch > 0:
        raise ValueError("invalid workspace size arguments")
    return int(n)


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, max_context,
           partition_tokens=512, out=None, out_dtype=None, workspace=None, stream=None):
    """Paged decode attention; returns ``out`` [batch, Hq, head_dim].

    ``out_dtype`` (default: q's dtype) may be torch.float32.  ``workspace`` is
    a uint8 CUDA buffer of ``decode_workspace_size(...)`` bytes (allocated here
    when not given).
    """
    dev = _device_tensors(("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                          ("block_tables", block_tables), ("context_lens", context_lens))
    batch, hq, d = q.shape
    if out is None:
        out = torch.empty((batch, hq, d), dtype=out_dtype or q.dtype, device=dev)
    if workspace is None:
        nbytes = decode_workspace_size(batch, hq, d, max_context, partition_tokens) if batch else 256
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _device_tensors(("out", out), ("workspace", workspace))
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_decode(ctypes.byref(_desc(q, "q")), ctypes.byref(_desc(k_cache, "k_cache")),
                           ctypes.byref(_desc(v_cache, "v_cache")),
                           ctypes.byref(_desc(block_tables, "block_tables")),
                           ctypes.byref(_desc(context_lens, "context_lens")), float(scale),
                           int(max_context), int(partition_tokens),
                           ctypes.byref(_desc(workspace, "workspace")), ctypes.byref(_desc(out, "out")),
                           _stream(dev, stream))
    _lib.check(rc, "pa_decode")
    return out


def decode_append(q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, scale, max_context,
                  partition_tokens=512, out=None, out_dtype=None, workspace=None, stream=None):
    """Store each sequence's new token (rows ``k_new[s]``, ``v_new[s]`` at
    position ``context_lens[s] - 1``) and run ``decode`` over the context that
    includes it, in one library call; same result as ``write_kv`` + ``decode``."""
    dev = _device_tensors(("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                          ("v_cache", v_cache), ("block_tables", block_tables), ("context_lens", context_lens))
    batch, hq, d = q.shape
    if out is None:
        out = torch.empty((batch, hq, d), dtype=out_dtype or q.dtype, device=dev)
    if workspace is None:
        nbytes = decode_workspace_size(batch, hq, d, max_context, partition_tokens) if batch else 256
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _device_tensors(("out", out), ("workspace", workspace))
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_decode_append(ctypes.byref(_desc(q, "q")), ctypes.byref(_desc(k_new, "k_new")),
                                  ctypes.byref(_desc(v_new, "v_new")), ctypes.byref(_desc(k_cache, "k_cache")),
                                  ctypes.byref(_desc(v_cache, "v_cache")),
                                  ctypes.byref(_desc(block_tables, "block_tables")),
                                  ctypes.byref(_desc(context_lens, "context_lens")), float(scale),
                                  int(max_context), int(partition_tokens),
                                  ctypes.byref(_desc(workspace, "workspace")), ctypes.byref(_desc(out, "out")),
                                  _stream(dev, stream))
    _lib.check(rc, "pa_decode_append")
    return out


def prefill_workspace_size(rows, num_q_heads, num_kv_heads, head_dim, batch, max_query_len, max_tokens) -> int:
    """Bytes of scratch ``prefill`` uses to split the keys of launches that
    would leave SMs idle (0 when it would not split)."""
    return int(library().pa_prefill_workspace_size(int(rows), int(num_q_heads), int(num_kv_heads), int(head_dim),
                                                   int(batch), int(max_query_len), int(max_tokens)))


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale, max_query_len,
            out=None, out_dtype=None, workspace=None, stream=None):
    """Causal attention of each sequence's new tokens over its paged context.

    ``q`` [rows, Hq, head_dim] packs the new tokens of all sequences; sequence
    ``s`` owns rows ``query_start[s] .. query_start[s+1]-1``, its last
    positions (their K/V already written to the cache).  ``workspace`` (uint8,
    ``prefill_workspace_size(...)`` bytes) lets a launch with few rows over
    long contexts split its keys; it is allocated here when needed and not
    given.  Returns ``out``.
    """
    dev = _device_tensors(("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                          ("block_tables", block_tables), ("context_lens", context_lens),
                          ("query_start", query_start))
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=dev)
    if workspace is None and q.shape[0] > 0 and max_query_len > 0:
        nbytes = prefill_workspace_size(q.shape[0], q.shape[1], k_cache.shape[1], q.shape[2], context_lens.shape[0],
                                        max_query_len, block_tables.shape[1] * k_cache.shape[2])
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _device_tensors(("out", out))
    if workspace is not None:
        _device_tensors(("workspace", workspace))
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_prefill(ctypes.byref(_desc(q, "q")), ctypes.byref(_desc(k_cache, "k_cache")),
                            ctypes.byref(_desc(v_cache, "v_cache")),
                            ctypes.byref(_desc(block_tables, "block_tables")),
                            ctypes.byref(_desc(context_lens, "context_lens")),
                            ctypes.byref(_desc(query_start, "query_start")), float(scale), int(max_query_len),
                            ctypes.byref(_desc(workspace, "workspace")) if workspace is not None else None,
                            ctypes.byref(_desc(out, "out")), _stream(dev, stream))
    _lib.check(rc, "pa_prefill")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale, max_context,
                   partition_tokens=512, out=None, stream=None):
    """``decode`` without a workspace: the library's built-in 32 MiB scratch is used.

    For callers that may not allocate device memory during decoding.  ``out``
    must then be passed in (a fresh one is allocated here only as a
    convenience).  Calls share the scratch, so order them on one stream.
    """
    dev = _device_tensors(("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                          ("block_tables", block_tables), ("context_lens", context_lens))
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    _device_tensors(("out", out))
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_decode_noalloc(ctypes.byref(_desc(q, "q")), ctypes.byref(_desc(k_cache, "k_cache")),
                                   ctypes.byref(_desc(v_cache, "v_cache")),
                                   ctypes.byref(_desc(block_tables, "block_tables")),
                                   ctypes.byref(_desc(context_lens, "context_lens")), float(scale),
                                   int(max_context), int(partition_tokens), ctypes.byref(_desc(out, "out")),
                                   _stream(dev, stream))
    _lib.check(rc, "pa_decode_noalloc")
    return out


def copy_blocks(caches, src_dst_pairs, stream=None):
    """Copy block pairs[i][0] onto pairs[i][1] in every cache."""
    caches = list(caches)
    dev = _device_tensors(("src_dst_pairs", src_dst_pairs), *[(f"caches[{i}]", c) for i, c in enumerate(caches)])
    arr = (_lib.PaTensor * max(1, len(caches)))()
    for i, c in enumerate(caches):
        arr[i] = _desc(c, f"caches[{i}]")
    lib = library()
    with torch.cuda.device(dev):
        rc = lib.pa_copy_blocks(arr, len(caches), ctypes.byref(_desc(src_dst_pairs, "src_dst_pairs")),
                                _stream(dev, stream))
    _lib.check(rc, "pa_copy_blocks")


def device_errors(stream=None, device=None) -> int:
    """Synchronise and return (and clear) the sticky device error bits."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        rc = library().pa_device_errors(_stream(dev, stream), ctypes.byref(bits))
    _lib.check(rc, "pa_device_errors")
    return int(bits.value)


def selftest_bounded_wait(polls: int = 1000, device=None) -> int:
    """Run the bounded-wait self-test kernel; returns the device error bits."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _lib.check(library().pa_selftest_bounded_wait(int(polls), _stream(dev, None)),
                   "pa_selftest_bounded_wait")
    return device_errors(device=dev)


def profile_enable(on: bool = True):
    """Record CUDA events around the main decode kernel of each pa_decode call."""
    _lib.check(library().pa_profile_enable(1 if on else 0), "pa_profile_enable")


def profile_take():
    """(summed milliseconds, number of recorded decode kernels) since the last take."""
    ms, n = ctypes.c_float(0.0), ctypes.c_int32(0)
    _lib.check(library().pa_profile_take(ctypes.byref(ms), ctypes.byref(n)), "pa_profile_take")
    return float(ms.value), int(n.value)


def read_probe(buf: torch.Tensor, sink: torch.Tensor, stream=None):
    """Stream ``buf`` (contiguous CUDA tensor, 16-byte aligned, a multiple of
    16 bytes) once and XOR its 32-bit words into ``sink`` (a one-element
    int32 CUDA tensor).  A measurement helper: timed over a buffer well above
    L2 it gives the read-only HBM rate the decode kernel is compared with."""
    if not (buf.is_cuda and sink.is_cuda) or buf.device != sink.device:
        raise ValueError("read_probe: buf and sink must be CUDA tensors on one device")
    if not buf.is_contiguous() or sink.dtype != torch.int32 or sink.numel() != 1:
        raise ValueError("read_probe: buf must be contiguous and sink a one-element int32 tensor")
    with torch.cuda.device(buf.device):
        _lib.check(library().pa_read_probe(ctypes.c_void_p(buf.data_ptr()),
                                           ctypes.c_uint64(buf.numel() * buf.element_size()),
                                           ctypes.c_void_p(sink.data_ptr()), _stream(buf.device, stream)),
                   "pa_read_probe")


def set_decode_path(path: int):
    """0 = automatic kernel choice, 1 = the generic CUDA-core kernel only."""
    _lib.check(library().pa_set_option(_lib.PA_OPT_DECODE_PATH, int(path)), "pa_set_option")


def get_decode_path() -> int:
    v = ctypes.c_int32(0)
    _lib.check(library().pa_get_option(_lib.PA_OPT_DECODE_PATH, ctypes.byref(v)), "pa_get_option")
    return int(v.value)


def set_prefill_path(path: int):
    """0 = automatic kernel choice, 1 = the generic CUDA-core prefill kernel only."""
    _lib.check(library().pa_set_option(_lib.PA_OPT_PREFILL_PATH, int(path)), "pa_set_option")


def get_prefill_path() -> int:
    v = ctypes.c_int32(0)
    _lib.check(library().pa_get_option(_lib.PA_OPT_PREFILL_PATH, ctypes.byref(v)), "pa_get_option")
    return int(v.value)


def set_checked(on: bool):
    """Checked mode: pa_write_kv, pa_copy_blocks and pa_decode_append first
    look for aliasing writes on the device, block the host, and raise (code
    PA_ERR_BOUNDS) instead of writing when they find one."""
    _lib.check(library().pa_set_option(_lib.PA_OPT_CHECKED, 1 if on else 0), "pa_set_option")


def get_checked() -> bool:
    v = ctypes.c_int32(0)
    _lib.check(library().pa_get_option(_lib.PA_OPT_CHECKED, ctypes.byref(v)), "pa_get_option")
    return bool(v.value)


def _i32_array(values):
    values = [int(x) for x in values]
    return (ctypes.c_int32 * max(1, len(values)))(*values), len(values)


class BlockPool:
    """Free pool + reference counts (``pa_alloc_*``)."""

    def __init__(self, num_blocks: int, init_free_order=None):
        self._lib = library()
        h = ctypes.c_void_p()
        if init_free_order is None:
            order_p = None
        else:
            arr, n = _i32_array(init_free_order)
            if n != num_blocks:
                raise ValueError("init_free_order must list every block once")
            order_p = arr
        _lib.check(self._lib.pa_alloc_create(int(num_blocks), order_p, ctypes.byref(h)), "pa_alloc_create")
        self._h = h
        self.num_blocks = int(num_blocks)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.pa_alloc_destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def alloc(self) -> int:
        b = ctypes.c_int32()
        _lib.check(self._lib.pa_alloc_block(self._h, ctypes.byref(b)), "pa_alloc_block")
        return b.value

    def incref(self, blocks, by: int = 1):
        arr, n = _i32_array(blocks)
        _lib.check(self._lib.pa_alloc_incref(self._h, arr, n, int(by)), "pa_alloc_incref")

    def decref(self, blocks):
        arr, n = _i32_array(blocks)
        _lib.check(self._lib.pa_alloc_decref(self._h, arr, n), "pa_alloc_decref")

    def cow(self, block: int):
        t, c = ctypes.c_int32(), ctypes.c_int32()
        _lib.check(self._lib.pa_alloc_cow(self._h, int(block), ctypes.byref(t), ctypes.byref(c)), "pa_alloc_cow")
        return t.value, bool(c.value)

    def refcount(self, block: int) -> int:
        r = ctypes.c_int32()
        _lib.check(self._lib.pa_alloc_refcount(self._h, int(block), ctypes.byref(r)), "pa_alloc_refcount")
        return r.value

    def refcounts(self):
        arr = (ctypes.c_int32 * max(1, self.num_blocks))()
        _lib.check(self._lib.pa_alloc_refcounts(self._h, arr, self.num_blocks), "pa_alloc_refcounts")
        return list(arr[: self.num_blocks])

    def num_free(self) -> int:
        n = ctypes.c_int32()
        _lib.check(self._lib.pa_alloc_num_free(self._h, ctypes.byref(n)), "pa_alloc_num_free")
        return n.value

    def stats(self) -> dict:
        """{num_blocks, free_blocks, used_blocks, shared_blocks, references}."""
        st = _lib.PaAllocStats()
        _lib.check(self._lib.pa_alloc_stats(self._h, ctypes.byref(st)), "pa_alloc_stats")
        return {name: int(getattr(st, name)) for name, _ in _lib.PaAllocStats._fields_}

    def free_list(self):
        n = self.num_free()
        arr = (ctypes.c_int32 * max(1, n))()
        got = ctypes.c_int32()
        _lib.check(self._lib.pa_alloc_free_list(self._h, arr, n, ctypes.byref(got)), "pa_alloc_free_list")
        return list(arr[: got.value])


class SequenceTables:
    """Per-sequence block tables on a BlockPool (``pa_seqs_*``)."""

    def __init__(self, pool: BlockPool, block_size: int = 16):
        self._lib = library()
        self.pool = pool           # keeps the pool alive
        self.block_size = int(block_size)
        h = ctypes.c_void_p()
        _lib.check(self._lib.pa_seqs_create(pool.handle, self.block_size, ctypes.byref(h)), "pa_seqs_create")
        self._h = h

    def snapshot(self) -> bytes:
        """The pool and every live table as bytes (``pa_seqs_snapshot``)."""
        n = ctypes.c_uint64()
        _lib.check(self._lib.pa_seqs_snapshot(self._h, None, 0, ctypes.byref(n)), "pa_seqs_snapshot")
        buf = ctypes.create_string_buffer(max(1, n.value))
        _lib.check(self._lib.pa_seqs_snapshot(self._h, buf, n.value, ctypes.byref(n)), "pa_seqs_snapshot")
        return buf.raw[: n.value]

    @classmethod
    def restore(cls, data: bytes) -> "SequenceTables":
        """A new pool and table set from ``snapshot()`` bytes (``pa_seqs_restore``)."""
        lib = library()
        buf = ctypes.create_string_buffer(bytes(data), max(1, len(data)))
        hp, hs = ctypes.c_void_p(), ctypes.c_void_p()
        _lib.check(lib.pa_seqs_restore(buf, len(data), ctypes.byref(hp), ctypes.byref(hs)), "pa_seqs_restore")
        pool = BlockPool.__new__(BlockPool)
        pool._lib, pool._h = lib, hp
        n = ctypes.c_int32()
        _lib.check(lib.pa_alloc_num_blocks(hp, ctypes.byref(n)), "pa_alloc_num_blocks")
        pool.num_blocks = n.value
        self = cls.__new__(cls)
        self._lib, self.pool, self._h = lib, pool, hs
        self.block_size = struct.unpack_from("=i", bytes(data), 12)[0]   # header word 3, native order
        return self

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.pa_seqs_destroy(h)
            self._h = None

    def add(self) -> int:
        s = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_add(self._h, ctypes.byref(s)), "pa_seqs_add")
        return s.value

    def append(self, seq_ids):
        """One token per listed sequence: (slots list, [(old, new) copy pairs])."""
        ids, n = _i32_array(seq_ids)
        slots = (ctypes.c_int32 * max(1, n))()
        pairs = (ctypes.c_int64 * max(2, 2 * n))()
        n_cow, n_done = ctypes.c_int32(), ctypes.c_int32()
        rc = self._lib.pa_seqs_append(self._h, ids, n, slots, pairs, ctypes.byref(n_cow), ctypes.byref(n_done))
        if rc != _lib.PA_OK:
            try:
                _lib.check(rc, "pa_seqs_append")
            except _lib.PagedKVError as e:
                e.done = n_done.value
                e.slots = list(slots[: n_done.value])
                e.pairs = [(pairs[2 * i], pairs[2 * i + 1]) for i in range(n_cow.value)]
                raise
        return list(slots[:n]), [(pairs[2 * i], pairs[2 * i + 1]) for i in range(n_cow.value)]

    def append_arrays(self, seq_ids):
        """Like ``append`` but returns (int32 slots tensor, int64 [P, 2] pairs tensor) on the host."""
        import numpy as np

        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
        n = len(ids)
        slots = np.empty(max(1, n), np.int32)
        pairs = np.empty((max(1, n), 2), np.int64)
        n_cow, n_done = ctypes.c_int32(), ctypes.c_int32()
        rc = self._lib.pa_seqs_append(
            self._h, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n,
            slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            pairs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), ctypes.byref(n_cow), ctypes.byref(n_done))
        _lib.check(rc, "pa_seqs_append")
        return torch.from_numpy(slots[:n]), torch.from_numpy(pairs[: n_cow.value])

    def append_n(self, seq: int, n_tokens: int):
        """Append a run of tokens to one sequence: (slots, copy pairs)."""
        slots = (ctypes.c_int32 * max(1, n_tokens))()
        pairs = (ctypes.c_int64 * max(2, 2 * n_tokens))()
        n_cow = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_append_n(self._h, int(seq), int(n_tokens), slots, pairs, ctypes.byref(n_cow)),
                   "pa_seqs_append_n")
        return list(slots[:n_tokens]), [(pairs[2 * i], pairs[2 * i + 1]) for i in range(n_cow.value)]

    def fork(self, parent: int) -> int:
        c = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_fork(self._h, int(parent), ctypes.byref(c)), "pa_seqs_fork")
        return c.value

    def free(self, seq: int):
        _lib.check(self._lib.pa_seqs_free(self._h, int(seq)), "pa_seqs_free")

    def length(self, seq: int) -> int:
        n = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_len(self._h, int(seq), ctypes.byref(n)), "pa_seqs_len")
        return n.value

    def table(self, seq: int):
        n = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_table(self._h, int(seq), None, 0, ctypes.byref(n)), "pa_seqs_table")
        arr = (ctypes.c_int32 * max(1, n.value))()
        _lib.check(self._lib.pa_seqs_table(self._h, int(seq), arr, n.value, ctypes.byref(n)), "pa_seqs_table")
        return list(arr[: n.value])

    def live(self):
        n = ctypes.c_int32()
        _lib.check(self._lib.pa_seqs_live(self._h, None, 0, ctypes.byref(n)), "pa_seqs_live")
        arr = (ctypes.c_int32 * max(1, n.value))()
        _lib.check(self._lib.pa_seqs_live(self._h, arr, n.value, ctypes.byref(n)), "pa_seqs_live")
        return list(arr[: n.value])

    def block_tables(self, seq_ids, max_blocks: int, pad: int = -1, out=None):
        """(int32 [n, max_blocks] tables, int32 [n] lengths) as host tensors.

        ``out`` = (tables, lens): contiguous int32 CPU tensors of those shapes
        (pinned buffers, say) to fill in place instead of allocating.
        """
        import numpy as np

        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
        n = len(ids)
        if out is not None:
            tables, lens = out
            if (tables.device.type != "cpu" or lens.device.type != "cpu" or tables.dtype != torch.int32
                    or lens.dtype != torch.int32 or tuple(tables.shape) != (n, max_blocks)
                    or tuple(lens.shape) != (n,) or not tables.is_contiguous() or not lens.is_contiguous()):
                raise ValueError("out must be contiguous int32 CPU tensors [n, max_blocks] and [n]")
            tp = ctypes.cast(tables.data_ptr(), ctypes.POINTER(ctypes.c_int32))
            lp = ctypes.cast(lens.data_ptr(), ctypes.POINTER(ctypes.c_int32))
        else:
            tables_np = np.empty((max(1, n), max(1, max_blocks)), np.int32)
            lens_np = np.empty(max(1, n), np.int32)
            tp = tables_np.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
            lp = lens_np.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        rc = self._lib.pa_seqs_block_tables(self._h, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n,
                                            int(max_blocks), int(pad), tp, lp)
        _lib.check(rc, "pa_seqs_block_tables")
        if out is not None:
            return out
        return torch.from_numpy(tables_np[:n, :max_blocks]), torch.from_numpy(lens_np[:n])
