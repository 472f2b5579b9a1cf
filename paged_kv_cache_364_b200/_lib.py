"""ctypes loader for ``libpagedkv.so`` and the ``pa_tensor`` descriptor.

The library is built in-tree (``paged_kv_cache_364_b200/build.py``).  If it is
missing, ``load()`` builds it with nvcc; if that is impossible it raises --
there is no fallback implementation of any kernel.
"""

from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpagedkv.so")

PA_OK = 0
PA_ERR_ARG = -1
PA_ERR_DTYPE = -2
PA_ERR_OOM = -3
PA_ERR_STATE = -4
PA_ERR_BOUNDS = -5
PA_ERR_CUDA = -6
PA_ERR_TIMEOUT = -7

PA_F32, PA_F16, PA_BF16, PA_I32, PA_I64, PA_U8 = range(6)

PA_DEVERR_BLOCK_ID = 1
PA_DEVERR_SLOT = 2
PA_DEVERR_CONTEXT_LEN = 4
PA_DEVERR_COPY_PAIR = 8
PA_DEVERR_WAIT_TIMEOUT = 16
PA_DEVERR_ALIAS = 32

PA_OPT_DECODE_PATH = 1
PA_OPT_PREFILL_PATH = 2
PA_OPT_CHECKED = 3

MAX_DIMS = 5


class PaTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("shape", ctypes.c_int64 * MAX_DIMS),
        ("stride", ctypes.c_int64 * MAX_DIMS),
    ]


class PaAllocStats(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int32),
        ("free_blocks", ctypes.c_int32),
        ("used_blocks", ctypes.c_int32),
        ("shared_blocks", ctypes.c_int32),
        ("references", ctypes.c_int64),
    ]


# Every symbol declared in include/pagedkv.h, with its ctypes signature.
_P = ctypes.POINTER
_T = _P(PaTensor)
_i32 = ctypes.c_int32
_i32p = _P(ctypes.c_int32)
_i64p = _P(ctypes.c_int64)
_u32p = _P(ctypes.c_uint32)
_vp = ctypes.c_void_p

SIGNATURES = {
    "pa_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_char_p, []),
    "pa_launch_count": (ctypes.c_int, [_P(ctypes.c_uint64)]),
    "pa_device_errors": (ctypes.c_int, [_vp, _u32p]),
    "pa_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, _vp]),
    "pa_write_kv": (ctypes.c_int, [_T, _T, _T, _T, _T, _vp]),
    "pa_decode_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32, _i32]),
    "pa_decode": (ctypes.c_int, [_T, _T, _T, _T, _T, ctypes.c_float, _i32, _i32, _T, _T, _vp]),
    "pa_decode_noalloc": (ctypes.c_int, [_T, _T, _T, _T, _T, ctypes.c_float, _i32, _i32, _T, _vp]),
    "pa_prefill": (ctypes.c_int, [_T, _T, _T, _T, _T, _T, ctypes.c_float, _i32, _T, _T, _vp]),
    "pa_prefill_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pa_decode_append": (ctypes.c_int, [_T, _T, _T, _T, _T, _T, _T, ctypes.c_float, _i32, _i32, _T, _T, _vp]),
    "pa_set_option": (ctypes.c_int, [_i32, _i32]),
    "pa_profile_enable": (ctypes.c_int, [_i32]),
    "pa_profile_take": (ctypes.c_int, [_P(ctypes.c_float), _i32p]),
    "pa_read_probe": (ctypes.c_int, [_vp, ctypes.c_uint64, _vp, _vp]),
    "pa_get_option": (ctypes.c_int, [_i32, _i32p]),
    "pa_copy_blocks": (ctypes.c_int, [_T, _i32, _T, _vp]),
    "pa_alloc_create": (ctypes.c_int, [_i32, _i32p, _P(_vp)]),
    "pa_alloc_destroy": (ctypes.c_int, [_vp]),
    "pa_alloc_block": (ctypes.c_int, [_vp, _i32p]),
    "pa_alloc_incref": (ctypes.c_int, [_vp, _i32p, _i32, _i32]),
    "pa_alloc_decref": (ctypes.c_int, [_vp, _i32p, _i32]),
    "pa_alloc_cow": (ctypes.c_int, [_vp, _i32, _i32p, _i32p]),
    "pa_alloc_refcount": (ctypes.c_int, [_vp, _i32, _i32p]),
    "pa_alloc_num_free": (ctypes.c_int, [_vp, _i32p]),
    "pa_alloc_num_blocks": (ctypes.c_int, [_vp, _i32p]),
    "pa_alloc_free_list": (ctypes.c_int, [_vp, _i32p, _i32, _i32p]),
    "pa_alloc_refcounts": (ctypes.c_int, [_vp, _i32p, _i32]),
    "pa_alloc_stats": (ctypes.c_int, [_vp, _P(PaAllocStats)]),
    "pa_seqs_create": (ctypes.c_int, [_vp, _i32, _P(_vp)]),
    "pa_seqs_destroy": (ctypes.c_int, [_vp]),
    "pa_seqs_add": (ctypes.c_int, [_vp, _i32p]),
    "pa_seqs_append": (ctypes.c_int, [_vp, _i32p, _i32, _i32p, _i64p, _i32p, _i32p]),
    "pa_seqs_append_n": (ctypes.c_int, [_vp, _i32, _i32, _i32p, _i64p, _i32p]),
    "pa_seqs_fork": (ctypes.c_int, [_vp, _i32, _i32p]),
    "pa_seqs_free": (ctypes.c_int, [_vp, _i32]),
    "pa_seqs_len": (ctypes.c_int, [_vp, _i32, _i32p]),
    "pa_seqs_table": (ctypes.c_int, [_vp, _i32, _i32p, _i32, _i32p]),
    "pa_seqs_live": (ctypes.c_int, [_vp, _i32p, _i32, _i32p]),
    "pa_seqs_block_tables": (ctypes.c_int, [_vp, _i32p, _i32, _i32, _i32, _i32p, _i32p]),
    "pa_seqs_snapshot": (ctypes.c_int, [_vp, _vp, ctypes.c_uint64, _P(ctypes.c_uint64)]),
    "pa_seqs_restore": (ctypes.c_int, [_vp, ctypes.c_uint64, _P(_vp), _P(_vp)]),
}

_lock = threading.Lock()
_lib = None


def _sources_newer_than(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    root = os.path.dirname(PKG)
    dirs = [os.path.join(PKG, "csrc"), os.path.join(root, "include")]
    for d in dirs:
        for f in os.listdir(d):
            if os.path.getmtime(os.path.join(d, f)) > t:
                return True
    return False


def load():
    """Load (building first if needed) the shared library; raise on failure."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if _sources_newer_than(LIB_PATH):
            from . import build as _build

            _build.build()
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


class PagedKVError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {detail} (code {code})")


class OutOfBlocks(PagedKVError):
    pass


class AllocatorStateError(PagedKVError):
    pass


def check(code: int, where: str):
    if code == PA_OK:
        return
    lib = load()
    detail = lib.pa_last_error().decode() or lib.pa_strerror(code).decode()
    if code == PA_ERR_OOM:
        raise OutOfBlocks(code, where, detail)
    if code == PA_ERR_STATE:
        raise AllocatorStateError(code, where, detail)
    raise PagedKVError(code, where, detail)
