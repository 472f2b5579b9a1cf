"""CPU oracle for the paged KV cache decode path.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
CPU restatement of what the GPU path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import it.  The product library
(``paged_kv_cache_364_b200``) never imports, links or calls anything here, and
nothing here imports the product library: the two share no code.

Modules
-------
attention   decode attention over a paged cache, in float64 (gather through the
            block table, then textbook softmax attention); partial states and
            the log-sum-exp merge used to pin the split-context identity.
cache_ops   bitwise slot-mapping writes and copy-on-write block copies.
allocator   free pool with reference counts, per-sequence block tables,
            append / fork / free / copy-on-write.

Sources (web pages on PagedAttention, cited by title and section):
  [SW]  "Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention"
  [PV]  "PagedAttention: How Virtual Memory Paging Solved LLM KV Cache Waste"
  [ML]  "49 vLLM / PagedAttention"

Every function is pinned by a test in ``tests/test_oracle_*.py`` against
something other than itself (brute force, closed forms, invariances, a library
routine, hand-worked fixtures under ``tests/golden/``).  No function here is
"parity unpinned".
"""

from . import allocator, attention, cache_ops  # noqa: F401

__all__ = ["allocator", "attention", "cache_ops"]
