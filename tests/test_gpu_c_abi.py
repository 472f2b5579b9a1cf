"""One decode step driven from plain C, with no Python or torch in the
process that computes it.

``tests/c_abi_decode.c`` is compiled with gcc against ``include/pagedkv.h``,
linked with ``libpagedkv.so`` and the CUDA runtime, and fed a seeded workload
from a file: it allocates device memory with cudaMalloc, stores each
sequence's new token with ``pa_write_kv`` and runs ``pa_decode`` (fast kernel,
several partitions, the in-kernel merge).  Its caches must equal the oracle's
append bit for bit and its fp32 output must be within the oracle tolerance.
"""

import os
import shutil
import struct
import subprocess

import numpy as np
import pytest
import torch

from gpu_util import assert_close_to_oracle, bits, needs_gpu
from oracle import attention as OA
from oracle import cache_ops as OC
from paged_kv_cache_364_b200 import _lib
from paged_kv_cache_364_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu, needs_gpu]
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
PA_DTYPE = {"fp32": 0, "fp16": 1, "bf16": 2}


@pytest.fixture(scope="module")
def decode_exe(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    _lib.load()
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path_factory.mktemp("c_abi") / "c_abi_decode")
    r = subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c_abi_decode.c"),
                        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                        "-L", libdir, "-lpagedkv", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                        f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("hq,hkv,d,dtype", [(32, 8, 128, "bf16"), (16, 16, 64, "fp16")])
def test_decode_step_from_c(decode_exe, tmp_path, hq, hkv, d, dtype):
    w = syn.custom_workload([1, 17, 300, 513, 2049, 5000], hq, hkv, d, dtype, seed=hq + d + 7)
    inp = syn.decode_inputs(w, "cpu")
    g = syn.generator(w.seed + 3, "cpu")
    k_new = syn.normal((w.batch, hkv, d), w.torch_dtype, "cpu", g)
    v_new = syn.normal((w.batch, hkv, d), w.torch_dtype, "cpu", g)
    tables = inp.block_tables.numpy().astype(np.int32)
    lens = inp.context_lens.numpy().astype(np.int32)
    slots = OC.last_token_slots(tables, w.lens, w.block_size).astype(np.int32)
    nb = inp.k_cache.shape[0]
    max_context = int(w.lens.max())
    path_in, path_out = str(tmp_path / "step.in"), str(tmp_path / "step.out")
    with open(path_in, "wb") as f:
        f.write(struct.pack("<9if", w.batch, hq, hkv, d, nb, tables.shape[1], PA_DTYPE[dtype], 512, max_context,
                            w.scale))
        for t in (inp.q, k_new, v_new, inp.k_cache, inp.v_cache):
            f.write(bits(t).tobytes())
        for a in (tables, lens, slots):
            f.write(np.ascontiguousarray(a).tobytes())
    r = subprocess.run([decode_exe, path_in, path_out], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr

    raw = open(path_out, "rb").read()
    n_out = w.batch * hq * d * 4
    cache_bytes = inp.k_cache.numel() * inp.k_cache.element_size()
    assert len(raw) == n_out + 2 * cache_bytes + 4
    out = np.frombuffer(raw[:n_out], dtype=np.float32).reshape(w.batch, hq, d)
    kc = np.frombuffer(raw[n_out:n_out + cache_bytes], dtype=np.int16).reshape(inp.k_cache.shape)
    vc = np.frombuffer(raw[n_out + cache_bytes:n_out + 2 * cache_bytes], dtype=np.int16).reshape(inp.k_cache.shape)
    errors = struct.unpack("<I", raw[-4:])[0]
    assert errors == 0

    want_k, want_v = OC.append_token(bits(k_new), bits(v_new), tables, w.lens, bits(inp.k_cache), bits(inp.v_cache))
    assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v)
    as_float = torch.from_numpy(np.ascontiguousarray(want_k)).view(w.torch_dtype)
    as_float_v = torch.from_numpy(np.ascontiguousarray(want_v)).view(w.torch_dtype)
    ref = OA.paged_decode(inp.q, as_float, as_float_v, tables, lens, w.scale)
    assert_close_to_oracle(torch.from_numpy(out.copy()), ref, w.torch_dtype, f"decode from C, {dtype}")
