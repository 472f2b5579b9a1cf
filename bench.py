#!/usr/bin/env python
"""Benchmark of the paged KV cache decode hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config gqa]
    python bench.py --impl reference ...      # the CPU oracle, timed as it stands

One step is one pass of the whole path over a batch: host allocator append of
one token per sequence (slot mapping, copy-on-write decisions), pa_copy_blocks
for any copy pairs, the store of the new tokens' K/V and the attention (plan,
split attention, log-sum-exp merge).  By default the store happens inside the
attention launch (pa_decode_append) and each step is replayed from a CUDA
graph; --append separate uses pa_write_kv + pa_decode, --launch eager launches
every kernel from the host.  The default workload is the batch-256 GQA
decode: 32 query / 8 KV heads, head_dim 128, bf16, block size 16, context lens
lognormal (median 1000, sigma 1, clipped to [16, 8192]), random physical block
placement, values N(0, 1).

Printed once by rank 0, one JSON line:
  value     KV-read GB/s of the whole step, inputs resident in HBM (algorithmic
            bytes: K and V of every attended token with each KV head counted
            once, plus q, out and block-table entries), max time over ranks.
  e2e       the same metric through the public API with per-step host->device
            copies of that step's inputs and a device->host read of the output.
  roofline  the split decode kernel alone: algorithmic bytes per launch over
            its CUDA-event duration, against the measured HBM copy peak.
  cpu_baseline  the float64 oracle on a bounded sample of the same workload.
  configs   (default gqa run on one GPU) the other workloads -- mha7b, long,
            cow (logical and unique bytes, the copy-on-write batch), tiny
            (latency) and prefill (TFLOP/s) -- each timed for a few steps
            with its own roofline and a bounded oracle sample.
Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch of
the same workload (own pool, own seed); no collective on the data path; the
timing is the max over ranks ("scaling": "weak").
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (% of HBM peak) and seq-steps/s"
UNIT = "GB/s"
STEP_STATES = 16          # distinct per-step metadata states, cycled (lengths grow <= 16 tokens)
FALLBACK_HBM_GBS = 6650.0

DESCRIPTIONS = {
    "gqa": "GQA decode: batch 256, 32 query / 8 KV heads, head_dim 128, bf16, block 16, context lens "
           "lognormal (median 1000, sigma 1.0) clipped to [16, 8192], random physical block placement",
    "mha7b": "7B-style MHA decode: batch 64, 32 heads, head_dim 128, fp16, block 16, context lens "
             "uniform in [128, 2048], pool = total blocks + 10% by random permutation",
    "long": "long-context split-context decode: batch 8, context lens uniform in [32768, 131072], "
            "32 query / 8 KV heads, head_dim 128, bf16, 512-token partitions merged by log-sum-exp",
    "tiny": "tiny decode: 4 seqs, lens {17, 33, 5, 64}, 4 heads (MHA), head_dim 64, fp32, pool of 32 blocks",
    "cow": "parallel sampling with prefix sharing + copy-on-write: 16 prompts x 1000 tokens shared by 8 samples "
           "(128 seqs, prompt blocks refcount 8), partial last prompt block copied on divergence, per-sample "
           "tails uniform in [0, 256]; 40 heads, head_dim 128, fp16, block 16",
    "prefill": "paged prefill: 32 requests, 32 query / 8 KV heads, head_dim 128, bf16, block 16; each request "
               "has a cached prefix uniform in [0, 2048] tokens and a chunk of new tokens uniform in [256, 2048] "
               "attended causally over prefix + chunk; random physical block placement",
    "chunked": "chunked prefill after long cached prefixes: 4 requests, 32 query / 8 KV heads, head_dim 128, bf16, "
               "block 16; prefixes uniform in [16384, 32768] tokens, chunks uniform in [64, 256] new tokens (the "
               "launch splits the keys); random physical block placement",
}
PREFILL_CONFIGS = ("prefill", "chunked")
PREFILL_METRIC = "paged prefill attention TFLOP/s (causal new tokens over the cached prefix)"
PREFILL_UNIT = "TFLOP/s"
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 << 20


# ------------------------------------------------------------------ setup ----
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="gqa", choices=sorted(DESCRIPTIONS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=48)
    ap.add_argument("--e2e-buffers", type=int, default=3, choices=(2, 3, 4),
                    help="input/output buffer sets of the end-to-end decode loop: with 3 the host prepares "
                         "step i while step i-1 runs and step i-2's output is still coming back")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--launch", choices=("graph", "eager"), default="graph",
                    help="replay each step from a CUDA graph captured per step state, or launch eagerly")
    ap.add_argument("--append", choices=("fused", "separate"), default="fused",
                    help="store the new token inside the attention launch (pa_decode_append) "
                         "or with its own pa_write_kv launch")
    ap.add_argument("--no-read-peak", action="store_true",
                    help="skip the same-run read-only ceiling (its 4 GiB buffer), e.g. under a profiler")
    ap.add_argument("--sweep", choices=("auto", "on", "off"), default="auto",
                    help="also time the other workloads (mha7b, long, cow, tiny, prefill, chunked) briefly and report "
                         "them under 'configs' (auto: with the default gqa workload on one GPU)")
    ap.add_argument("--sweep-steps", type=int, default=20)
    ap.add_argument("--sweep-warmup", type=int, default=5)
    ap.add_argument("--sweep-cpu-seconds", type=float, default=4.0)
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str, timeout_s: float = 120.0):
    """One process per GPU.  The short timeout makes a collective fail with an
    error, rather than wait for good, when another rank has died."""
    if world > 1 and not torch.distributed.is_initialized():
        import datetime

        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))


def reduce_max(x: float, world: int, device) -> float:
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device) -> float:
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch of the same workload (weak scaling)."""
    return base_seed + 1000 * rank


def measured_peaks(key="hbm_gbs"):
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return float(mp[key]), "measured"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}[key], "fallback"


# -------------------------------------------------------------- workload ----
def algorithmic_bytes(lens, w) -> int:
    """Bytes a decode step must move: K+V of attended tokens (each KV head once),
    q, out and the block-table entries read."""
    lens = np.asarray(lens, np.int64)
    kv = int(lens.sum()) * 2 * w.n_kv_heads * w.head_dim * w.elt_bytes
    qo = 2 * w.batch * w.n_q_heads * w.head_dim * w.elt_bytes
    tables = int((-(-lens // w.block_size)).sum()) * 4
    return kv + qo + tables


class StepStates:
    """Per-step metadata produced by the product allocator, for STEP_STATES steps.

    Sequence s starts with lens[s] - 1 tokens placed (their K/V are the random
    pool contents, as after a prefill), so the first step attends lens[s]
    tokens.  Each step appends one token per sequence; the states are cycled so
    the workload's length distribution holds for any number of steps.
    """

    def __init__(self, w, device, n_states=STEP_STATES):
        import paged_kv_cache_364_b200 as pk

        # The workload's pool, plus headroom for the tokens the bench appends
        # after the measured step (the step states and the end-to-end steps):
        # the extra ids sit at the bottom of the free stack, so every block
        # the workload's own steps take comes from its own pool first.
        headroom_tokens = n_states + 64
        self.num_blocks = w.num_blocks + w.batch * (-(-headroom_tokens // w.block_size) + 1)
        order = np.concatenate([np.arange(w.num_blocks, self.num_blocks), w.placement]).astype(np.int64)
        self.pool = pk.BlockPool(self.num_blocks, order)
        self.seqs = pk.SequenceTables(self.pool, w.block_size)
        self.ids = []
        self.cow_pairs = []          # copy-on-write pairs made before the measured steps
        if w.name == "cow":
            self._build_sharing(w)
        else:
            for n in w.lens:
                s = self.seqs.add()
                if n > 1:
                    self.seqs.append_n(s, int(n) - 1)
                self.ids.append(s)
        self.max_blocks = int(-(-(int(w.lens.max()) + n_states + 64) // w.block_size))
        slots, tables, lens, pairs = [], [], [], []
        for _ in range(n_states):
            sl, pr = self.seqs.append_arrays(self.ids)
            tb, ln = self.seqs.block_tables(self.ids, self.max_blocks)
            slots.append(sl)
            tables.append(tb)
            lens.append(ln)
            pairs.append(pr.to(device) if len(pr) else None)
        self.slots = torch.stack(slots).to(device)
        self.tables = torch.stack(tables).to(device)
        self.lens = torch.stack(lens).to(device)
        self.lens_host = torch.stack(lens).numpy()
        self.pairs = pairs
        self.max_context = int(self.lens_host.max())
        self.n = n_states

    def _build_sharing(self, w):
        """Prompts, forks into samples, then per-sample tails in sample order."""
        from paged_kv_cache_364_b200 import synthetic as syn

        shape = syn.CowShape(seed=w.seed)
        tails = syn.cow_tails(w.seed, shape.n_prompts, shape.n_samples).ravel()
        for _ in range(shape.n_prompts):
            p = self.seqs.add()
            self.seqs.append_n(p, shape.prompt_len)
            self.ids.append(p)
            self.ids.extend(self.seqs.fork(p) for _ in range(shape.n_samples - 1))
        for r in range(int(tails.max())):
            active = [s for i, s in enumerate(self.ids) if tails[i] > r]
            _, pairs = self.seqs.append(active)
            self.cow_pairs.extend(pairs)

    def unique_kv_bytes(self, j, w):
        """K+V bytes of the distinct physical blocks read in step j (shared blocks once)."""
        tables = self.tables[j].cpu().numpy()
        blocks = set()
        for i, n in enumerate(self.lens_host[j]):
            blocks.update(tables[i, : -(-int(n) // w.block_size)].tolist())
        return len(blocks) * w.block_size * 2 * w.n_kv_heads * w.head_dim * w.elt_bytes


# ------------------------------------------------------------------ clocks ----
def nvml_handle(nv, cuda_index: int):
    """(NVML handle, how it was found) for CUDA device ``cuda_index`` as this
    process numbers it.  CUDA_VISIBLE_DEVICES renumbers CUDA devices but not
    NVML's, so the device is matched by UUID, then PCI bus id, and only then
    by index."""
    props = None
    try:
        props = torch.cuda.get_device_properties(cuda_index)
    except Exception:
        pass
    if props is not None:
        try:
            uuid = str(props.uuid)
            if uuid:
                return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid), "uuid"
        except Exception:
            pass
        try:
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus), "pci"
        except Exception:
            pass
    return nv.nvmlDeviceGetHandleByIndex(cuda_index), "index"


class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons, power) in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        self.ok = False
        self.matched_by = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h, self.matched_by = nvml_handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((mhz, int(reasons)))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml" if self.ok else "unavailable"}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "source": "nvml", "device_matched_by": self.matched_by}


# ------------------------------------------------------------- our arm ------
def run_ours(args, rank, world, local, sub=False, read_peak=None):
    """The decode step of ``args.config``.  ``sub``: a short entry of the
    workload sweep -- no end-to-end loop, and the read-only ceiling of the
    headline run (``read_peak``) instead of a new measurement."""
    import paged_kv_cache_364_b200 as pk
    from paged_kv_cache_364_b200 import synthetic as syn

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    base = syn.workload(args.config)
    w = syn.workload(args.config, seed=rank_seed(base.seed, rank))
    st = StepStates(w, device)
    gen = syn.generator(w.seed, device)
    dt = w.torch_dtype
    kc = syn.random_cache(st.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    vc = syn.random_cache(st.num_blocks, w.n_kv_heads, w.block_size, w.head_dim, dt, device, gen)
    qs = syn.normal((st.n, w.batch, w.n_q_heads, w.head_dim), dt, device, gen)
    ks = syn.normal((st.n, w.batch, w.n_kv_heads, w.head_dim), dt, device, gen)
    vs = syn.normal((st.n, w.batch, w.n_kv_heads, w.head_dim), dt, device, gen)
    part = w.partition_tokens
    ws = torch.empty(pk.decode_workspace_size(w.batch, w.n_q_heads, w.head_dim, st.max_context, part),
                     dtype=torch.uint8, device=device)
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=dt, device=device)
    stream = torch.cuda.current_stream(device)
    cow = None
    if st.cow_pairs:
        pairs = torch.tensor(st.cow_pairs, dtype=torch.int64, device=device)
        pk.copy_blocks([kc, vc], pairs)        # warm
        torch.cuda.synchronize()
        reps = 20                               # back to back, so host issue time is hidden
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(reps):
            pk.copy_blocks([kc, vc], pairs)
        c1.record(stream)
        c1.synchronize()
        copy_bytes = 2 * 2 * len(st.cow_pairs) * w.n_kv_heads * w.block_size * w.head_dim * w.elt_bytes
        ms = c0.elapsed_time(c1) / reps
        cow = {"pairs": len(st.cow_pairs), "copy_ms": round(ms, 4), "bytes_read_plus_written": copy_bytes,
               "GBps": round(copy_bytes / (ms * 1e-3) / 1e9, 1)}

    def step(i):
        j = i % st.n
        if st.pairs[j] is not None:
            pk.copy_blocks([kc, vc], st.pairs[j])
        if args.append == "fused":
            pk.decode_append(qs[j], ks[j], vs[j], kc, vc, st.tables[j], st.lens[j], w.scale, st.max_context,
                             part, out=out, workspace=ws)
            return
        pk.write_kv(ks[j], vs[j], st.slots[j], kc, vc)
        pk.decode(qs[j], kc, vc, st.tables[j], st.lens[j], w.scale, st.max_context, part,
                  out=out, workspace=ws)

    graphs = None
    launches_per_graph = 0
    if args.launch == "graph":
        # one graph per step state (the states differ in their metadata buffers)
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for j in range(st.n):
                step(j)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        n0 = pk.launch_count()
        for j in range(st.n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(j)
            graphs.append(g)
        launches_per_graph = (pk.launch_count() - n0) // st.n
        eager_step = step

        def step(i):  # noqa: F811 - replay instead of eager launches
            graphs[i % st.n].replay()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    pk.profile_enable(True)
    pk.profile_take()
    launches0 = pk.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    pk.profile_enable(False)
    launches = pk.launch_count() - launches0
    if graphs is not None:
        launches = launches_per_graph * args.steps
    split_ms, split_n = pk.profile_take()
    if graphs is not None:
        # kernel-only timing of the split kernel, measured on eager steps
        pk.profile_enable(True)
        for i in range(min(args.steps, 200)):
            eager_step(i)
        torch.cuda.synchronize()
        pk.profile_enable(False)
        split_ms, split_n = pk.profile_take()
    elapsed_ms = e0.elapsed_time(e1)
    errors = pk.device_errors()

    step_idx = [(args.warmup + i) % st.n for i in range(args.steps)]
    bytes_rank = float(sum(algorithmic_bytes(st.lens_host[j], w) for j in step_idx))
    max_ms = reduce_max(elapsed_ms, world, device)
    total_bytes = reduce_sum(bytes_rank, world, device)
    total_seq_steps = reduce_sum(float(w.batch * args.steps), world, device)
    split_avg_ms = split_ms / max(split_n, 1)
    split_bytes = bytes_rank / max(args.steps, 1)

    # ---- end to end: host allocator + pinned H2D inputs + D2H output, per step
    e2e = None if sub else run_e2e(args, w, st, kc, vc, ws, part, device, gen, world)
    if read_peak is None and not args.no_read_peak:
        read_peak = measure_read_peak(device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, st, kc, vc, qs, args.cpu_seconds)
    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    traffic = profiled_traffic(args.config)
    value = total_bytes / (max_ms * 1e-3) / 1e9
    achieved = split_bytes / (split_avg_ms * 1e-3) / 1e9 if split_n else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"bf16": "bf16", "fp16": "fp16", "fp32": "f32"}[w.dtype],
        "data": "synthetic",
        "config": {
            "workload": DESCRIPTIONS[args.config],
            "name": args.config,
            "batch_per_gpu": w.batch,
            "global_batch": int(w.batch * world),
            "q_heads": w.n_q_heads,
            "kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim,
            "block_size": w.block_size,
            "partition_tokens": part,
            "mean_context": float(np.mean(st.lens_host)),
            "kv_bytes_per_step": int(np.mean([algorithmic_bytes(st.lens_host[j], w) for j in range(st.n)])),
            "parallelism": f"dp{world} (independent sequence batches, no collective)",
            "l2": l2_note(int(np.mean([algorithmic_bytes(st.lens_host[j], w) for j in range(st.n)]))),
            "cuda_graph": args.launch == "graph",
            "append": args.append,
        },
        "seq_steps_per_s": round(total_seq_steps / (max_ms * 1e-3), 1),
        # sequences per second of the attention kernel alone (its average launch)
        "decode_only_seq_steps_per_s": round(w.batch * world / (split_avg_ms * 1e-3), 1) if split_n else None,
        "pct_of_hbm_peak": round(100.0 * value / world / peak, 2),
        "pct_of_8tbps_nominal": round(100.0 * value / world / 8000.0, 2),
        "pct_of_read_peak_same_run": round(100.0 * value / world / read_peak["value"], 2) if read_peak else None,
        "read_peak_same_run": read_peak,
        "roofline": {
            "kernel": "decode_fast_kernel (split attention)",
            "bound": "hbm",
            "achieved": round(achieved, 2) if achieved else None,
            "peak": peak,
            "peak_source": f"{peak_kind}: MEASURED_PEAKS.json hbm_gbs (copy)" if peak_kind == "measured"
                           else "fallback 6650 GB/s",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4) if achieved else None,
            "traffic": traffic,
            "avg_launch_ms": round(split_avg_ms, 6),
            "launches_timed": split_n,
            # DRAM bytes of the profiled launch over this run's launch time:
            # below the algorithmic rate when shared pages are re-read from L2
            "dram_achieved": round(traffic / (split_avg_ms * 1e-3) / 1e9, 2) if traffic and split_n else None,
            # the kernel only reads K/V, so also against this GPU's read-only streaming rate
            "frac_of_read_peak": round(achieved / read_peak["value"], 4) if achieved and read_peak else None,
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        "copy_on_write": cow,
        "unique_kv_bytes_per_step": (int(np.mean([st.unique_kv_bytes(j, w) for j in range(st.n)]))
                                     if w.name == "cow" else None),
        "gpu_launches": int(launches),
        "device_errors": errors,
        "clocks": sampler.summary(),
    }
    return line


def l2_note(step_bytes: int) -> str:
    if step_bytes > 4 * L2_BYTES:
        return f"no flush: every step reads {step_bytes / 1e9:.2f} GB of K/V, far above the 126 MB L2"
    return (f"no flush: a step reads {step_bytes / 1e6:.2f} MB, which stays in the 126 MB L2 between steps "
            f"(a latency figure, not an HBM one)")


SWEEP = ("mha7b", "long", "cow", "tiny", "prefill", "chunked")
# what each sweep entry keeps from its workload's full line
SWEEP_KEYS = ("metric", "value", "unit", "ms_per_step", "steps", "warmup", "dtype", "seq_steps_per_s",
              "decode_only_seq_steps_per_s", "pct_of_hbm_peak", "pct_of_8tbps_nominal",
              "pct_of_read_peak_same_run", "roofline", "cpu_baseline", "copy_on_write", "unique_kv_bytes_per_step",
              "gpu_launches", "device_errors", "clocks")


def run_sweep(args, rank, world, local, read_peak):
    """The other workloads of the decode path (and prefill), each timed for a
    few steps after the headline run, on one GPU.  Each entry is the same
    measurement as that workload's own ``--config`` run, without the
    end-to-end loop; the tiny workload is a latency figure."""
    import argparse as _ap

    out = {}
    for name in SWEEP:
        sub = _ap.Namespace(**vars(args))
        sub.config, sub.steps, sub.warmup = name, args.sweep_steps, args.sweep_warmup
        sub.cpu_seconds = args.sweep_cpu_seconds
        torch.cuda.empty_cache()
        if name in PREFILL_CONFIGS:
            line = run_prefill(sub, rank, world, local, sub=True)
        else:
            line = run_ours(sub, rank, world, local, sub=True, read_peak=read_peak)
        entry = {k: line.get(k) for k in SWEEP_KEYS if k in line}
        entry["workload"] = DESCRIPTIONS[name]
        entry["config"] = line["config"]
        if name == "tiny":
            entry["latency_us_per_step"] = round(line["ms_per_step"] * 1e3, 2)
            entry["note"] = "the pool fits in L2: a latency figure; the GB/s and roofline fields are not HBM figures"
        if name == "cow":
            lb = line["config"]["kv_bytes_per_step"]
            ub = line.get("unique_kv_bytes_per_step")
            entry["logical_kv_bytes_per_step"] = lb
            entry["unique_GBps"] = round(ub / (line["ms_per_step"] * 1e-3) / 1e9, 2) if ub else None
        out[name] = entry
    return out


def measure_read_peak(device, nbytes=4 << 30, reps=10):
    """Read-only HBM rate of this GPU in this run: pa_read_probe over a 4 GiB
    buffer (32x L2), 3 warm-up launches, then ``reps`` launches timed with
    CUDA events on the launching stream."""
    import paged_kv_cache_364_b200 as pk

    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        pk.read_probe(buf, sink)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        pk.read_probe(buf, sink)
    e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del buf
    torch.cuda.empty_cache()
    return {"value": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "kernel": "read_probe_kernel (16-byte read-only loads, 4 in flight per thread, 1024 threads per SM)",
            "bytes": nbytes, "launches": reps}


def run_e2e(args, w, st, kc, vc, ws, part, device, gen, world):
    """Public-API steps with per-step pinned host->device inputs and a
    device->host output, pipelined as a serving loop would run them: inputs
    and outputs rotate over ``--e2e-buffers`` sets, host->device and
    device->host copies run on two streams of their own, and the host prepares
    step i (allocator append, block tables, H2D) while the GPU runs step i-1.
    Before reusing a buffer set the host reads the output that set last
    carried, so with two sets the chain "output of step i-2 back, host work,
    inputs of step i over" must fit inside one kernel; a third set takes it
    off the critical path.  The timed region ends when the last output is
    back."""
    import paged_kv_cache_364_b200 as pk
    from paged_kv_cache_364_b200 import synthetic as syn

    nbuf = args.e2e_buffers
    # at least one step past the buffer sets; the step states leave 64 tokens of table headroom
    K = max(3, nbuf + 1, min(args.e2e_steps, 48))
    dt = w.torch_dtype
    fused = args.append == "fused"
    q_h = syn.normal((K, w.batch, w.n_q_heads, w.head_dim), dt, device, gen).cpu().pin_memory()
    k_h = syn.normal((K, w.batch, w.n_kv_heads, w.head_dim), dt, device, gen).cpu().pin_memory()
    v_h = syn.normal((K, w.batch, w.n_kv_heads, w.head_dim), dt, device, gen).cpu().pin_memory()

    def pinned(shape, dtype):
        return [torch.empty(shape, dtype=dtype).pin_memory() for _ in range(nbuf)]

    def dev(shape, dtype):
        return [torch.empty(shape, dtype=dtype, device=device) for _ in range(nbuf)]

    tables_h, lens_h = pinned((w.batch, st.max_blocks), torch.int32), pinned((w.batch,), torch.int32)
    slots_h = pinned((w.batch,), torch.int32)
    out_h = pinned((w.batch, w.n_q_heads, w.head_dim), dt)
    q_d, k_d, v_d = (dev((w.batch, w.n_q_heads, w.head_dim), dt), dev((w.batch, w.n_kv_heads, w.head_dim), dt),
                     dev((w.batch, w.n_kv_heads, w.head_dim), dt))
    tables_d, lens_d, slots_d = dev((w.batch, st.max_blocks), torch.int32), dev((w.batch,), torch.int32), \
        dev((w.batch,), torch.int32)
    out_d = dev((w.batch, w.n_q_heads, w.head_dim), dt)
    stream = torch.cuda.current_stream(device)
    copy = torch.cuda.Stream(device)          # host -> device
    back = torch.cuda.Stream(device)          # device -> host, kept apart so the next step's inputs
                                              # never queue behind this step's output
    h2d_ev = [torch.cuda.Event() for _ in range(nbuf)]
    run_ev = [torch.cuda.Event() for _ in range(nbuf)]
    d2h_ev = [torch.cuda.Event() for _ in range(nbuf)]
    pending = [None] * nbuf                  # step whose output sits in buffer b, not yet read
    e2e_max_context = st.max_context + K + 16
    ws2 = torch.empty(pk.decode_workspace_size(w.batch, w.n_q_heads, w.head_dim, e2e_max_context, part),
                      dtype=torch.uint8, device=device)
    acc = {"h2d": 0, "d2h": 0, "checksum": 0.0}
    lens_seen = []                           # per-step lengths, for the byte count after timing
    graphs = None                            # per buffer set: the step's kernels as one CUDA graph

    def launch(b):
        if fused:
            pk.decode_append(q_d[b], k_d[b], v_d[b], kc, vc, tables_d[b], lens_d[b], w.scale, e2e_max_context, part,
                             out=out_d[b], workspace=ws2)
        else:
            pk.write_kv(k_d[b], v_d[b], slots_d[b], kc, vc)
            pk.decode(q_d[b], kc, vc, tables_d[b], lens_d[b], w.scale, e2e_max_context, part, out=out_d[b],
                      workspace=ws2)

    def collect(b):
        if pending[b] is not None:
            d2h_ev[b].synchronize()          # this step's output is on the host: read it
            acc["checksum"] += float(out_h[b][0, 0, 0])
            acc["d2h"] += out_h[b].numel() * out_h[b].element_size()
            pending[b] = None

    def step(i):
        b = i % nbuf
        collect(b)                           # buffer b free again (step i - 2 finished)
        slots, pairs = st.seqs.append_arrays(st.ids)
        st.seqs.block_tables(st.ids, st.max_blocks, out=(tables_h[b], lens_h[b]))
        with torch.cuda.stream(copy):
            sent = [(q_d[b], q_h[i]), (k_d[b], k_h[i]), (v_d[b], v_h[i]), (tables_d[b], tables_h[b]),
                    (lens_d[b], lens_h[b])]
            if not fused:
                slots_h[b].copy_(slots)
                sent.append((slots_d[b], slots_h[b]))
            for d_, h_ in sent:
                d_.copy_(h_, non_blocking=True)
            h2d_ev[b].record(copy)
        nbytes = sum(h_.numel() * h_.element_size() for _, h_ in sent)
        stream.wait_event(h2d_ev[b])
        if len(pairs):
            pr = pairs.pin_memory().to(device, non_blocking=True)
            nbytes += pr.numel() * 8
            pk.copy_blocks([kc, vc], pr)
        if graphs is not None:
            graphs[b].replay()
        else:
            launch(b)
        run_ev[b].record(stream)
        with torch.cuda.stream(back):
            back.wait_event(run_ev[b])
            out_h[b].copy_(out_d[b], non_blocking=True)
            d2h_ev[b].record(back)
        pending[b] = i
        acc["h2d"] += nbytes
        lens_seen.append(lens_h[b].numpy().copy())

    for i in range(nbuf):                    # warm the path, every buffer set once
        step(i)
    for b in range(nbuf):
        collect(b)
    torch.cuda.synchronize()
    if args.launch == "graph":
        graphs = []
        for b in range(nbuf):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                launch(b)
            graphs.append(g)
        torch.cuda.synchronize()
    acc.update(h2d=0, d2h=0)
    lens_seen.clear()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy.wait_event(e0)
    back.wait_event(e0)
    for i in range(nbuf, K):
        step(i)
    for b in range(nbuf):
        collect(b)
    stream.wait_stream(copy)
    stream.wait_stream(back)
    e1.record(stream)
    e1.synchronize()
    ms = reduce_max(e0.elapsed_time(e1), world, device)
    total = reduce_sum(float(sum(algorithmic_bytes(ln, w) for ln in lens_seen)), world, device)
    n = max(K - nbuf, 1)
    del graphs
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": UNIT,
            "h2d_bytes_per_step": int(acc["h2d"] / n), "d2h_bytes_per_step": int(acc["d2h"] / n),
            "ms_per_step": round(ms / n, 4), "steps": n,
            "includes": ("host allocator append + block tables into pinned buffers, H2D of q/k/v/tables/lens"
                         + ("" if fused else "/slots") + " on a copy stream, copy + "
                         + ("fused append-and-decode" if fused else "write + decode") + " kernels, D2H of out "
                         f"read on the host; {nbuf} buffer sets so step i's host work and copies overlap "
                         "step i-1's kernels" + ("; each buffer set's kernels replayed from a CUDA graph"
                                            if args.launch == "graph" else ""))}


def cpu_baseline(w, st, kc, vc, qs, seconds):
    """The float64 oracle, as it stands, on as many sequences as fit the budget."""
    from oracle import attention as OA

    j = 0
    tables = st.tables[j].cpu().numpy()
    lens = st.lens_host[j]
    q = qs[j].cpu()
    k_host, v_host = kc.cpu(), vc.cpu()
    t0 = time.perf_counter()
    done, nbytes = 0, 0
    while done < w.batch and (time.perf_counter() - t0 < seconds or done < 4):
        OA.paged_decode_rows(q, k_host, v_host, tables, lens, w.scale, [done])
        nbytes += int(lens[done]) * 2 * w.n_kv_heads * w.head_dim * w.elt_bytes
        done += 1
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": UNIT, "cores": threads_used(),
            "kind": "oracle", "seq_steps_per_s": round(done / dt, 3),
            "cpu_count": os.cpu_count(), "nproc": len(os.sched_getaffinity(0)),
            "sample": f"first {done} of {w.batch} sequences of one step ({nbytes / 1e9:.3f} GB of K/V), "
                      f"{dt:.1f} s, float64 NumPy oracle"}


def threads_used() -> int:
    n = torch.get_num_threads()
    try:
        from threadpoolctl import threadpool_info

        n = max([n] + [int(i.get("num_threads", 1)) for i in threadpool_info()])
    except Exception:
        pass
    return int(n)


def profiled_traffic(config: str, profile: str | None = None, source: str = "decode.cu"):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, when that summary was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", profile or f"decode_split_{config}_ncu.md")
    src = os.path.join(ROOT, "paged_kv_cache_364_b200", "csrc", source)
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        vals = {}
        for line in open(path):
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip()
        if vals.get(f"{source} sha256 prefix") != digest:
            return None
        return int(float(vals["dram_bytes_per_launch"]))
    except Exception:
        return None


# ------------------------------------------------------- reference arm ------
def run_reference(args, rank, world):
    """The CPU oracle on a bounded sample of the same workload, per step."""
    if rank != 0:
        return None
    from oracle import attention as OA
    from paged_kv_cache_364_b200 import synthetic as syn

    w = syn.workload(args.config)
    budget_s = 150.0                       # whole reference run, warm-up included
    # calibrate on one sequence, then take as many sequences per step as fit
    one = syn.custom_workload(w.lens[:1], w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype, w.block_size,
                              w.partition_tokens, seed=w.seed, extra_blocks=0)
    one_inp = syn.decode_inputs(one, "cpu")
    t0 = time.perf_counter()
    OA.paged_decode(one_inp.q, one_inp.k_cache, one_inp.v_cache, one_inp.block_tables.numpy(), one.lens,
                    one.scale)
    t_one = max(time.perf_counter() - t0, 1e-4)
    per_step = int(max(1, min(w.batch, budget_s / ((args.steps + args.warmup) * t_one))))
    rows = list(range(per_step))
    sub_lens = w.lens[rows]
    sw = syn.custom_workload(sub_lens, w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype, w.block_size,
                             w.partition_tokens, seed=w.seed, extra_blocks=0)
    inp = syn.decode_inputs(sw, "cpu")
    tables = inp.block_tables.numpy()

    def step():
        OA.paged_decode(inp.q, inp.k_cache, inp.v_cache, tables, sw.lens, sw.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    kv = int(sw.lens.sum()) * 2 * sw.n_kv_heads * sw.head_dim * sw.elt_bytes
    value = kv * args.steps / dt / 1e9
    sample = (f"first {per_step} of {w.batch} sequences per step ({kv / 1e9:.4f} GB of K/V), "
              f"float64 NumPy oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": DESCRIPTIONS[args.config], "name": args.config},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- prefill ----
def prefill_flops(lens, qlens, w) -> int:
    """Useful flops of a prefill step: every (new token, visible key, query
    head) pair costs 2d for q.k and 2d for p.v; masked keys are not counted."""
    pairs = sum(int(q) * (int(n) - int(q)) + int(q) * (int(q) + 1) // 2 for n, q in zip(lens, qlens))
    return pairs * w.n_q_heads * 4 * w.head_dim


def prefill_slots(w, tables) -> np.ndarray:
    """Cache slots of every new token (positions n - q_len .. n - 1), host side."""
    out = []
    for s, (n, q) in enumerate(zip(w.lens, w.qlens)):
        for pos in range(int(n - q), int(n)):
            out.append(int(tables[s, pos // w.block_size]) * w.block_size + pos % w.block_size)
    return np.asarray(out, np.int32)


def run_prefill(args, rank, world, local, sub=False):
    """One step = store the new tokens' K/V (pa_write_kv) + pa_prefill over the
    paged cache.  ``sub``: a short entry of the workload sweep (no end-to-end loop)."""
    import paged_kv_cache_364_b200 as pk
    from paged_kv_cache_364_b200 import synthetic as syn

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    base = syn.workload(args.config)
    w = syn.workload(args.config, seed=rank_seed(base.seed, rank))
    inp = syn.prefill_inputs(w, device)
    gen = syn.generator(w.seed + 1, device)
    rows = int(w.qlens.sum())
    k_new = syn.normal((rows, w.n_kv_heads, w.head_dim), w.torch_dtype, device, gen)
    v_new = syn.normal((rows, w.n_kv_heads, w.head_dim), w.torch_dtype, device, gen)
    slots = torch.from_numpy(prefill_slots(w, inp.block_tables.cpu().numpy())).to(device)
    out = torch.empty(inp.q.shape, dtype=inp.q.dtype, device=device)
    mq = int(w.qlens.max())
    stream = torch.cuda.current_stream(device)

    def attend():
        pk.prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start, w.scale,
                   mq, out=out)

    def step():
        pk.write_kv(k_new, v_new, slots, inp.k_cache, inp.v_cache)
        attend()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    sampler = ClockSampler(local)
    launches0 = pk.launch_count()
    with sampler:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        e1.synchronize()
    barrier(world)
    launches = pk.launch_count() - launches0
    elapsed_ms = e0.elapsed_time(e1)
    # the attention kernel alone, on the stream it is launched on
    k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_k = max(1, min(args.steps, 50))
    k0.record(stream)
    for _ in range(n_k):
        attend()
    k1.record(stream)
    k1.synchronize()
    kernel_ms = k0.elapsed_time(k1) / n_k
    errors = pk.device_errors()

    flops = prefill_flops(w.lens, w.qlens, w)
    max_ms = reduce_max(elapsed_ms, world, device)
    total = reduce_sum(float(flops) * args.steps, world, device)
    e2e = None if sub else run_prefill_e2e(args, w, inp, k_new, v_new, slots, device, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = prefill_cpu_baseline(w, inp, args.cpu_seconds)
    if rank != 0:
        return None
    clocks = sampler.summary()
    # the kernel-only timing runs right after the long timed loop: when that
    # loop ran under the power cap, the sustained GEMM figure is the peak
    capped = "sw_power_cap" in clocks.get("reasons", [])
    peak_key = "bf16_tflops_sustained" if capped else "bf16_tflops"
    peak, peak_kind = measured_peaks(peak_key)
    value = total / (max_ms * 1e-3) / 1e12
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    return {
        "metric": PREFILL_METRIC,
        "value": round(value, 2),
        "unit": PREFILL_UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": DESCRIPTIONS[args.config],
            "name": args.config,
            "requests_per_gpu": w.batch,
            "new_tokens_per_step": rows,
            "mean_context": float(np.mean(w.lens)),
            "q_heads": w.n_q_heads,
            "kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim,
            "block_size": w.block_size,
            "flops_per_step": int(flops),
            "parallelism": f"dp{world} (independent request batches, no collective)",
            "l2": (f"no flush: every step reads {inp.q.numel() * 2 / 1e9:.2f} GB of queries and a "
                   f"{2 * inp.k_cache.numel() * 2 / 1e9:.2f} GB K/V pool, above the 126 MB L2"),
        },
        "roofline": {
            "kernel": ("prefill_tc_kernel (tcgen05, causal)" if args.config == "prefill"
                       else "prefill_tc_kernel with key split + prefill_merge_kernel"),
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_source": (f"{peak_kind}: MEASURED_PEAKS.json {peak_key} (cuBLAS bf16 GEMM, "
                            f"{'sustained: the timed loop ran under sw_power_cap' if capped else 'burst'})"
                            if peak_kind == "measured"
                            else f"fallback {peak:g} TFLOP/s ({'sustained' if capped else 'burst'})"),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            # DRAM bytes per launch of the prefill kernel (with the key split, the
            # split kernel alone: 95 % of the step; the merge kernel is not counted)
            "traffic": profiled_traffic(args.config, f"prefill_tc_{args.config}_ncu.md", "prefill.cu"),
            "avg_launch_ms": round(kernel_ms, 6),
            "launches_timed": n_k,
            "note": "flops count visible (new token, key) pairs only; the kernel also multiplies the masked "
                    "half of diagonal tiles and a second 16-bit term of each softmax weight",
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "device_errors": errors,
        "clocks": clocks,
    }


def run_prefill_e2e(args, w, inp, k_new, v_new, slots, device, world):
    """Through the public API with host buffers: every step copies its new
    tokens (q, k, v), slots, tables, lengths and starts from pinned host
    memory and reads its output back on the host.  Pipelined like the decode
    loop: inputs and outputs double-buffered, H2D and D2H on separate copy
    streams, so step i's input copies overlap step i-1's kernels and output."""
    import paged_kv_cache_364_b200 as pk

    K = max(3, min(args.e2e_steps, 8))
    names = ("q", "k", "v", "slots", "tables", "lens", "starts")
    host = {n: t.cpu().pin_memory() for n, t in zip(names, (inp.q, k_new, v_new, slots, inp.block_tables,
                                                             inp.context_lens, inp.query_start))}
    nbuf = 2
    dev = [{n: torch.empty_like(t, device=device) for n, t in host.items()} for _ in range(nbuf)]
    out_d = [torch.empty_like(inp.q) for _ in range(nbuf)]
    out_h = [torch.empty(inp.q.shape, dtype=inp.q.dtype).pin_memory() for _ in range(nbuf)]
    stream = torch.cuda.current_stream(device)
    copy, back = torch.cuda.Stream(device), torch.cuda.Stream(device)
    h2d_ev = [torch.cuda.Event() for _ in range(nbuf)]
    run_ev = [torch.cuda.Event() for _ in range(nbuf)]
    d2h_ev = [torch.cuda.Event() for _ in range(nbuf)]
    pending = [False] * nbuf
    mq = int(w.qlens.max())
    checksum = 0.0

    def collect(b):
        nonlocal checksum
        if pending[b]:
            d2h_ev[b].synchronize()
            checksum += float(out_h[b][0, 0, 0])
            pending[b] = False

    def step(i):
        b = i % nbuf
        collect(b)
        d = dev[b]
        with torch.cuda.stream(copy):
            for n in names:
                d[n].copy_(host[n], non_blocking=True)
            h2d_ev[b].record(copy)
        stream.wait_event(h2d_ev[b])
        pk.write_kv(d["k"], d["v"], d["slots"], inp.k_cache, inp.v_cache)
        pk.prefill(d["q"], inp.k_cache, inp.v_cache, d["tables"], d["lens"], d["starts"], w.scale, mq, out=out_d[b])
        run_ev[b].record(stream)
        with torch.cuda.stream(back):
            back.wait_event(run_ev[b])
            out_h[b].copy_(out_d[b], non_blocking=True)
            d2h_ev[b].record(back)
        pending[b] = True

    for i in range(2):
        step(i)
    for b in range(nbuf):
        collect(b)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy.wait_event(e0)
    back.wait_event(e0)
    for i in range(K):
        step(i)
    for b in range(nbuf):
        collect(b)
    stream.wait_stream(copy)
    stream.wait_stream(back)
    e1.record(stream)
    e1.synchronize()
    ms = reduce_max(e0.elapsed_time(e1), world, device)
    total = reduce_sum(float(prefill_flops(w.lens, w.qlens, w)) * K, world, device)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    return {"value": round(total / (ms * 1e-3) / 1e12, 3), "unit": PREFILL_UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(out_h[0].numel() * out_h[0].element_size()), "ms_per_step": round(ms / K, 3),
            "steps": K, "includes": "pinned H2D of q/k/v/slots/tables/lens/starts on a copy stream, write + "
                                    "prefill kernels, D2H of out on a second copy stream read on the host; "
                                    "double-buffered so copies overlap the neighbouring steps"}


def prefill_cpu_baseline(w, inp, seconds):
    """The float64 prefill oracle, as it stands, on whole sequences until the budget is spent."""
    from oracle import attention as OA

    q, kc, vc = inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu()
    tables, lens, starts = inp.block_tables.cpu(), inp.context_lens.cpu(), inp.query_start.cpu()
    order = list(np.argsort(w.qlens))              # shortest chunks first, so the sample spans several requests
    t0 = time.perf_counter()
    done = []
    while len(done) < len(order) and (time.perf_counter() - t0 < seconds or not done):
        s = int(order[len(done)])
        OA.paged_prefill(q, kc, vc, tables, lens, starts, w.scale, seqs=[s])
        done.append(s)
    dt = time.perf_counter() - t0
    flops = prefill_flops(w.lens[done], w.qlens[done], w)
    return {"value": round(flops / dt / 1e12, 6), "unit": PREFILL_UNIT, "cores": threads_used(), "kind": "oracle",
            "sample": f"{len(done)} of {w.batch} requests (the shortest new-token chunks, "
                      f"{int(w.qlens[done].sum())} rows), {dt:.1f} s, float64 NumPy oracle"}


def run_prefill_reference(args, rank, world):
    """The float64 prefill oracle on a bounded sample of the workload, per step."""
    if rank != 0:
        return None
    from oracle import attention as OA
    from paged_kv_cache_364_b200 import synthetic as syn

    w = syn.workload(args.config)
    # a sample of whole requests small enough that the run stays within minutes
    s = int(np.argmin(w.qlens))
    sw = syn.custom_prefill(w.lens[[s]], w.qlens[[s]], w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype,
                            seed=w.seed, extra_blocks=0)
    inp = syn.prefill_inputs(sw, "cpu")
    t0 = time.perf_counter()
    OA.paged_prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                     sw.scale)
    t_one = max(time.perf_counter() - t0, 1e-3)
    rows = max(1, int(sw.qlens[0] * min(1.0, 150.0 / ((args.steps + args.warmup) * t_one))))
    sw = syn.custom_prefill([int(sw.lens[0] - sw.qlens[0] + rows)], [rows], w.n_q_heads, w.n_kv_heads,
                            w.head_dim, w.dtype, seed=w.seed, extra_blocks=0)
    inp = syn.prefill_inputs(sw, "cpu")

    def step():
        OA.paged_prefill(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, inp.query_start,
                         sw.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = prefill_flops(sw.lens, sw.qlens, sw) * args.steps / dt / 1e12
    sample = (f"one request per step: {rows} new tokens after a {int(sw.lens[0]) - rows}-token prefix "
              f"(the workload's shortest chunk, trimmed to the time budget), float64 NumPy oracle")
    return {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": PREFILL_UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCRIPTIONS[args.config], "name": args.config},
        "cpu_baseline": {"value": round(value, 6), "unit": PREFILL_UNIT, "cores": threads_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": PREFILL_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = (run_prefill_reference if args.config in PREFILL_CONFIGS else run_reference)(args, rank, world)
    elif args.config in PREFILL_CONFIGS:
        line = run_prefill(args, rank, world, local)
    else:
        line = run_ours(args, rank, world, local)
        sweep = args.sweep == "on" or (args.sweep == "auto" and args.config == "gqa" and world == 1)
        if sweep and world == 1 and line is not None:
            line["configs"] = run_sweep(args, rank, world, local, line["read_peak_same_run"])
    if line is not None and rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
