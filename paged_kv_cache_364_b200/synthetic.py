"""Seeded synthetic inputs for the paged decode workloads.

This module only draws numbers: context lengths, pool sizes, a random physical
placement of blocks, and N(0, 1) tensors cast to the workload's dtype.  It holds
none of the method's arithmetic (no slot computation, no attention, no
allocator policy), so the tests can hand the same inputs to the CUDA path and to
the CPU oracle.  It imports neither of them.

Workloads (sizes of the decode step on one layer):

  tiny    4 sequences, lens {17, 33, 5, 64}, 4 heads (MHA), head_dim 64, fp32,
          pool of 32 blocks, placement = first 10 ids of a seeded permutation.
  mha7b   batch 64, 32 heads (MHA), head_dim 128, fp16, lens uniform in
          [128, 2048], pool = total blocks + 10 %, permuted placement.
  gqa     batch 256, 32 query / 8 KV heads, head_dim 128, bf16, lens lognormal
          (median 1000, sigma 1.0 in log space) clipped to [16, 8192].
  cow     16 prompts x 1000 tokens, 8 samples each (128 sequences), per-sample
          tails uniform in [0, 256]; 40 heads (MHA), head_dim 128, fp16; pool =
          exact need + 10 %.  Sharing and copy-on-write are built by the caller
          through the allocator (lens here = prompt + tail + 1).
  long    batch 8, lens uniform in [32768, 131072], 32 query / 8 KV heads,
          head_dim 128, bf16, 512-token partitions.
  prefill 32 requests, 32 query / 8 KV heads, head_dim 128, bf16; each has a
          cached prefix uniform in [0, 2048] tokens and a chunk of new tokens
          uniform in [256, 2048] (lens = prefix + new tokens); random placement.
  chunked 4 requests, same heads; cached prefixes uniform in [16384, 32768]
          and chunks uniform in [64, 256] tokens (few rows over long contexts).

Values are N(0, 1) drawn in fp32 by a seeded ``torch.Generator`` on the target
device, then cast; lengths and placements come from ``numpy.random.default_rng``
with the same seed.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16

DTYPES = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class DecodeWorkload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str
    block_size: int
    lens: np.ndarray                  # int64 [batch], tokens attended per sequence
    num_blocks: int
    partition_tokens: int
    seed: int
    placement: np.ndarray = field(default=None)   # int64 permutation of the pool

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def elt_bytes(self) -> int:
        return torch.tensor([], dtype=self.torch_dtype).element_size()

    def blocks_per_seq(self) -> np.ndarray:
        return -(-self.lens // self.block_size)

    def kv_bytes(self) -> int:
        """K+V bytes of the attended tokens (each KV head counted once)."""
        return int(self.lens.sum()) * 2 * self.n_kv_heads * self.head_dim * self.elt_bytes


@dataclass
class PrefillWorkload(DecodeWorkload):
    qlens: np.ndarray = field(default=None)     # int64 [batch], new tokens per sequence (<= lens)

    def query_start(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.qlens)]).astype(np.int32)


def _pool_size(total_blocks: int) -> int:
    return int(math.ceil(1.1 * total_blocks))


def workload(name: str, seed: int | None = None, batch: int | None = None) -> DecodeWorkload:
    """The named decode workload with its lengths and placement drawn."""
    default_seed = {"tiny": 1, "mha7b": 2, "gqa": 3, "cow": 4, "long": 5, "prefill": 6, "chunked": 7}[name]
    seed = default_seed if seed is None else seed
    rng = np.random.default_rng(seed)
    B = BLOCK_SIZE
    if name == "tiny":
        lens = np.array([17, 33, 5, 64], np.int64)
        w = DecodeWorkload(name, 4, 4, 4, 64, "fp32", B, lens, 32, 512, seed)
    elif name == "mha7b":
        n = 64 if batch is None else batch
        lens = rng.integers(128, 2048, size=n, endpoint=True).astype(np.int64)
        nb = _pool_size(int((-(-lens // B)).sum()))
        w = DecodeWorkload(name, n, 32, 32, 128, "fp16", B, lens, nb, 512, seed)
    elif name == "gqa":
        n = 256 if batch is None else batch
        z = rng.standard_normal(n)
        lens = np.clip(np.round(np.exp(math.log(1000.0) + 1.0 * z)), 16, 8192).astype(np.int64)
        nb = _pool_size(int((-(-lens // B)).sum()))
        w = DecodeWorkload(name, n, 32, 8, 128, "bf16", B, lens, nb, 512, seed)
    elif name == "cow":
        shape = CowShape(seed=seed)
        tails = cow_tails(seed, shape.n_prompts, shape.n_samples).ravel()
        # tokens attended by each sample in the measured step: prompt + tail + new token
        lens = (shape.prompt_len + tails + 1).astype(np.int64)
        prompt_blocks = -(-shape.prompt_len // B)
        own = -(-(shape.prompt_len % B + tails + 1) // B)   # the copied partial block onwards
        need = shape.n_prompts * prompt_blocks + int(own.sum())
        w = DecodeWorkload(name, len(lens), shape.n_heads, shape.n_heads, shape.head_dim, shape.dtype, B, lens,
                           _pool_size(need), 512, seed)
    elif name == "long":
        n = 8 if batch is None else batch
        lens = rng.integers(32768, 131072, size=n, endpoint=True).astype(np.int64)
        nb = _pool_size(int((-(-lens // B)).sum()))
        w = DecodeWorkload(name, n, 32, 8, 128, "bf16", B, lens, nb, 512, seed)
    elif name == "prefill":
        n = 32 if batch is None else batch
        prefix = rng.integers(0, 2048, size=n, endpoint=True).astype(np.int64)
        qlens = rng.integers(256, 2048, size=n, endpoint=True).astype(np.int64)
        lens = prefix + qlens
        nb = _pool_size(int((-(-lens // B)).sum()))
        w = PrefillWorkload(name, n, 32, 8, 128, "bf16", B, lens, nb, 512, seed, qlens=qlens)
    elif name == "chunked":
        n = 4 if batch is None else batch
        prefix = rng.integers(16384, 32768, size=n, endpoint=True).astype(np.int64)
        qlens = rng.integers(64, 256, size=n, endpoint=True).astype(np.int64)
        lens = prefix + qlens
        nb = _pool_size(int((-(-lens // B)).sum()))
        w = PrefillWorkload(name, n, 32, 8, 128, "bf16", B, lens, nb, 512, seed, qlens=qlens)
    else:
        raise KeyError(name)
    w.placement = rng.permutation(w.num_blocks).astype(np.int64)
    return w


def custom_prefill(lens, qlens, n_q_heads, n_kv_heads, head_dim, dtype, block_size=BLOCK_SIZE, seed=0,
                   extra_blocks=7) -> PrefillWorkload:
    """A prefill workload: sequence s holds lens[s] tokens, the last qlens[s] of them new."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int64)
    qlens = np.asarray(qlens, np.int64)
    nb = int((-(-lens // block_size)).sum()) + extra_blocks
    w = PrefillWorkload("custom", len(lens), n_q_heads, n_kv_heads, head_dim, dtype, block_size, lens, nb, 512,
                        seed, qlens=qlens)
    w.placement = rng.permutation(nb).astype(np.int64)
    return w


def custom_workload(lens, n_q_heads, n_kv_heads, head_dim, dtype, block_size=BLOCK_SIZE,
                    partition_tokens=512, seed=0, extra_blocks=7) -> DecodeWorkload:
    """A decode workload with the given context lengths and head shapes."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int64)
    nb = int((-(-lens // block_size)).sum()) + extra_blocks
    w = DecodeWorkload("custom", len(lens), n_q_heads, n_kv_heads, head_dim, dtype, block_size,
                       lens, nb, partition_tokens, seed)
    w.placement = rng.permutation(nb).astype(np.int64)
    return w


def placement_tables(w: DecodeWorkload, pad: int = -1) -> np.ndarray:
    """Block tables from consecutive ids of the seeded permutation.

    Sequence order, then logical block order; unused entries hold ``pad``.
    Returns int32 ``[batch, max_blocks]``.
    """
    nbs = w.blocks_per_seq()
    max_blocks = int(nbs.max()) if len(nbs) else 1
    tables = np.full((w.batch, max(max_blocks, 1)), pad, np.int32)
    pos = 0
    for s, nb in enumerate(nbs):
        tables[s, :nb] = w.placement[pos:pos + nb]
        pos += nb
    return tables


def normal(shape, dtype, device, generator: torch.Generator) -> torch.Tensor:
    """N(0, 1) drawn in fp32 then cast (values are the cast bits)."""
    return torch.randn(shape, generator=generator, device=device, dtype=torch.float32).to(dtype)


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def random_cache(num_blocks, n_kv_heads, block_size, head_dim, dtype, device, gen,
                 chunk_blocks: int = 4096) -> torch.Tensor:
    """A pool [NB, Hkv, B, d] filled with N(0, 1) values, drawn chunk by chunk."""
    out = torch.empty((num_blocks, n_kv_heads, block_size, head_dim), dtype=dtype, device=device)
    for b0 in range(0, num_blocks, chunk_blocks):
        b1 = min(num_blocks, b0 + chunk_blocks)
        out[b0:b1] = normal((b1 - b0, n_kv_heads, block_size, head_dim), dtype, device, gen)
    return out


@dataclass
class DecodeInputs:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor


def decode_inputs(w: DecodeWorkload, device="cpu") -> DecodeInputs:
    """q and a fully populated pool for one decode step of workload ``w``."""
    gen = generator(w.seed, device)
    dt = w.torch_dtype
    k_cache = random_cache(w.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    v_cache = random_cache(w.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    q = normal((w.batch, w.n_q_heads, w.head_dim), dt, device, gen)
    tables = torch.from_numpy(placement_tables(w)).to(device)
    lens = torch.from_numpy(w.lens.astype(np.int32)).to(device)
    return DecodeInputs(q, k_cache, v_cache, tables, lens)


@dataclass
class PrefillInputs:
    q: torch.Tensor                   # [rows, Hq, d], the new tokens of all sequences packed
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    query_start: torch.Tensor         # int32 [batch + 1]


def prefill_inputs(w: PrefillWorkload, device="cpu") -> PrefillInputs:
    """Query rows and a fully populated pool for one prefill step of ``w``."""
    gen = generator(w.seed, device)
    dt = w.torch_dtype
    k_cache = random_cache(w.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    v_cache = random_cache(w.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    q = normal((int(w.qlens.sum()), w.n_q_heads, w.head_dim), dt, device, gen)
    tables = torch.from_numpy(placement_tables(w)).to(device)
    lens = torch.from_numpy(w.lens.astype(np.int32)).to(device)
    starts = torch.from_numpy(w.query_start()).to(device)
    return PrefillInputs(q, k_cache, v_cache, tables, lens, starts)


def cow_tails(seed: int = 4, n_prompts: int = 16, n_samples: int = 8) -> np.ndarray:
    """Per-sample tail lengths (uniform in [0, 256]) for the sharing workload."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(n_prompts, n_samples), endpoint=True).astype(np.int64)


@dataclass
class CowShape:
    n_prompts: int = 16
    prompt_len: int = 1000
    n_samples: int = 8
    n_heads: int = 40
    head_dim: int = 128
    dtype: str = "fp16"
    block_size: int = BLOCK_SIZE
    seed: int = 4
