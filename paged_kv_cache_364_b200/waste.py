"""KV-memory utilisation: contiguous reservation versus paged blocks.

The pages contrast two ways of holding the KV cache of concurrent requests
("Stop Wasting GPU Memory: A Deep Dive Into vLLM's PagedAttention", TL;DR and
Technical Details; "49 vLLM / PagedAttention", "Paging for the KV cache: where
the x2-4 comes from"):

* contiguous: each admitted request reserves one contiguous range sized for
  its prompt plus the maximum output length, because the real output length is
  unknown.  Unused tail slots are internal waste; free ranges too small for the
  next request are external waste (holes).
* paged: blocks of B slots are taken from a free pool as the sequence grows, so
  at most B - 1 slots of the last block are unused.

``simulate`` runs one seeded request trace through both schemes on the same
token-slot budget and reports, averaged over the decode steps, the fraction of
the pool that holds real tokens, the internal and external waste, and the
number of requests decoded concurrently (a larger effective batch is where the
serving speed-up of paging comes from).  The paged side uses the library's C++
allocator (``pa_seqs_*``); the contiguous side is a first-fit range allocator.
All numbers are for synthetic traces; they reproduce the kind of comparison the
pages report, not their figures.

    python -m paged_kv_cache_364_b200.waste [--pool-tokens N] [--requests R]
"""

from __future__ import annotations

import argparse
import json
import math
from dataclasses import dataclass, field

import numpy as np


@dataclass
class Trace:
    prompt: np.ndarray          # tokens per request
    output: np.ndarray          # generated tokens per request
    max_output: int             # what a contiguous scheme must reserve


def lognormal_trace(n_requests=2000, seed=0, prompt_median=400, output_median=250, sigma=1.0,
                    max_output=2048, max_prompt=4096) -> Trace:
    """Seeded request lengths: lognormal prompts and outputs, clipped."""
    rng = np.random.default_rng(seed)
    prompt = np.clip(np.round(np.exp(math.log(prompt_median) + sigma * rng.standard_normal(n_requests))),
                     16, max_prompt).astype(np.int64)
    output = np.clip(np.round(np.exp(math.log(output_median) + sigma * rng.standard_normal(n_requests))),
                     1, max_output).astype(np.int64)
    return Trace(prompt, output, max_output)


class FirstFit:
    """Contiguous ranges over [0, size): first-fit allocation, coalescing free."""

    def __init__(self, size: int):
        self.size = size
        self.free = [(0, size)]          # sorted (start, length)

    def alloc(self, n: int):
        for i, (st, ln) in enumerate(self.free):
            if ln >= n:
                if ln == n:
                    self.free.pop(i)
                else:
                    self.free[i] = (st + n, ln - n)
                return st
        return None

    def release(self, st: int, n: int):
        self.free.append((st, n))
        self.free.sort()
        merged = []
        for s, l in self.free:
            if merged and merged[-1][0] + merged[-1][1] == s:
                merged[-1] = (merged[-1][0], merged[-1][1] + l)
            else:
                merged.append((s, l))
        self.free = merged

    def largest_hole(self) -> int:
        return max((l for _, l in self.free), default=0)

    def free_total(self) -> int:
        return sum(l for _, l in self.free)


@dataclass
class Stats:
    steps: int = 0
    used: float = 0.0            # sum over steps of tokens held
    reserved: float = 0.0        # sum over steps of slots reserved by running requests
    external: float = 0.0        # sum over steps of free slots unusable by the next request
    batch: float = 0.0           # sum over steps of running requests
    finished: int = 0
    samples: list = field(default_factory=list)

    def summary(self, pool: int) -> dict:
        s = max(self.steps, 1)
        return {
            "utilisation": self.used / (s * pool),
            "internal_waste": (self.reserved - self.used) / (s * pool),
            "external_waste": self.external / (s * pool),
            "mean_batch": self.batch / s,
            "finished": self.finished,
            "steps": self.steps,
            "preemptions": len(self.samples),
        }


def run_contiguous(trace: Trace, pool: int, max_steps: int) -> Stats:
    ff = FirstFit(pool)
    queue = list(range(len(trace.prompt)))
    running = {}                          # rid -> (start, reserved, length)
    st = Stats()
    for _ in range(max_steps):
        while queue:                      # admit in order while the next one fits
            rid = queue[0]
            need = int(trace.prompt[rid] + trace.max_output)
            start = ff.alloc(need)
            if start is None:
                break
            queue.pop(0)
            running[rid] = (start, need, int(trace.prompt[rid]))
        if not running:
            break
        done = []
        for rid, (start, need, length) in running.items():
            length += 1
            running[rid] = (start, need, length)
            if length >= trace.prompt[rid] + trace.output[rid]:
                done.append(rid)
        st.steps += 1
        st.used += sum(v[2] for v in running.values())
        st.reserved += sum(v[1] for v in running.values())
        nxt = int(trace.prompt[queue[0]] + trace.max_output) if queue else None
        st.external += ff.free_total() if (nxt is not None and ff.largest_hole() < nxt) else 0
        st.batch += len(running)
        for rid in done:
            start, need, _ = running.pop(rid)
            ff.release(start, need)
            st.finished += 1
    return st


def run_paged(trace: Trace, pool: int, max_steps: int, block_size: int = 16) -> Stats:
    """Blocks on demand from the library allocator; when a step needs more
    blocks than are free, the newest running request is preempted (its blocks
    freed, the request re-queued from its prompt), as a serving engine does."""
    import paged_kv_cache_364_b200 as pk

    nb = pool // block_size
    bp = pk.BlockPool(nb)
    seqs = pk.SequenceTables(bp, block_size)
    queue = list(range(len(trace.prompt)))
    running = {}                          # rid -> seq id, in admission order
    length = {}
    watermark = max(1, nb // 100)
    st = Stats()
    for _ in range(max_steps):
        while queue:                      # admit while the prompt fits above the watermark
            rid = queue[0]
            need_blocks = -(-int(trace.prompt[rid]) // block_size) + 1
            if bp.num_free() - need_blocks < watermark:
                break
            queue.pop(0)
            sid = seqs.add()
            seqs.append_n(sid, int(trace.prompt[rid]))
            running[rid] = sid
            length[rid] = int(trace.prompt[rid])
        if not running:
            break
        need = sum(1 for r in running if length[r] % block_size == 0)
        while need > bp.num_free() and running:
            victim = next(reversed(running))
            seqs.free(running.pop(victim))
            need -= 1 if length[victim] % block_size == 0 else 0
            queue.insert(0, victim)
            st.samples.append(victim)     # preemptions
        done = []
        ids = list(running.values())
        if ids:
            seqs.append(ids)
        for rid in running:
            length[rid] += 1
            if length[rid] >= trace.prompt[rid] + trace.output[rid]:
                done.append(rid)
        st.steps += 1
        st.used += sum(length[r] for r in running)
        # slots the allocator holds for running requests (no block is shared here)
        st.reserved += bp.stats()["used_blocks"] * block_size
        st.batch += len(running)
        for rid in done:
            seqs.free(running.pop(rid))
            st.finished += 1
    return st


def simulate(pool_tokens=1 << 20, n_requests=20000, seed=0, max_steps=2000, block_size=16, **trace_kw) -> dict:
    """Both schemes on one trace.  The defaults keep both request queues
    non-empty for every step, so the averages describe a saturated server
    rather than the drain at the end of a finite trace."""
    trace = lognormal_trace(n_requests, seed, **trace_kw)
    c = run_contiguous(trace, pool_tokens, max_steps).summary(pool_tokens)
    p = run_paged(trace, pool_tokens, max_steps, block_size).summary(pool_tokens)
    return {"pool_tokens": pool_tokens, "requests": n_requests, "block_size": block_size,
            "max_output_reserved": trace.max_output, "contiguous": c, "paged": p,
            "batch_gain": p["mean_batch"] / max(c["mean_batch"], 1e-9)}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--pool-tokens", type=int, default=1 << 20)
    ap.add_argument("--requests", type=int, default=20000)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--block-size", type=int, default=16)
    a = ap.parse_args(argv)
    print(json.dumps(simulate(a.pool_tokens, a.requests, a.seed, a.steps, a.block_size), indent=1))


if __name__ == "__main__":
    main()
