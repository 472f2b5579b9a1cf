"""Host-side logic of bench.py on CPU: byte accounting, the multi-rank
reductions over a world-size-2 gloo group, and the reference (oracle) arm."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_cache_364_b200 import synthetic as syn  # noqa: E402


def test_algorithmic_bytes_counts_each_kv_head_once():
    w = syn.workload("gqa")
    got = bench.algorithmic_bytes(w.lens, w)
    kv = int(w.lens.sum()) * 2 * 8 * 128 * 2
    qo = 2 * 256 * 32 * 128 * 2
    tables = int((-(-w.lens // 16)).sum()) * 4
    assert got == kv + qo + tables
    assert 1.5e9 < kv < 2.0e9


def test_rank_seeds_are_distinct_and_stable():
    seeds = [bench.rank_seed(3, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == 3
    a = syn.workload("gqa", seed=seeds[1])
    b = syn.workload("gqa", seed=seeds[1])
    assert np.array_equal(a.lens, b.lens)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, wsz, _ = bench.dist_env()
    bench.dist_init(wsz, "gloo")
    dev = torch.device("cpu")
    bench.barrier(wsz)
    mx = bench.reduce_max(10.0 + r, wsz, dev)         # per-rank elapsed ms
    sm = bench.reduce_sum(1000.0 * (r + 1), wsz, dev)  # per-rank bytes
    bench.barrier(wsz)
    q.put((r, mx, sm))
    torch.distributed.destroy_process_group()


def test_two_rank_reductions_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 11.0, 3000.0), (1, 11.0, 3000.0)]


def _dying_worker(rank, world, port, q):
    """Rank 1 leaves between steps (after the first reduction); rank 0's next
    reduction must end with an error instead of waiting for it."""
    import time

    import torch

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.dist_init(world, "gloo", timeout_s=5.0)
    dev = torch.device("cpu")
    bench.reduce_max(1.0, world, dev)
    if rank == 1:
        os._exit(0)                                   # gone, with no collective in flight
    t0 = time.time()
    try:
        bench.reduce_max(2.0, world, dev)
        q.put((rank, "no error", time.time() - t0))
    except Exception as e:                            # noqa: BLE001 - any error is the signal
        q.put((rank, type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()                                   # flush the queue's feeder thread before _exit
    os._exit(0)


def test_a_rank_that_leaves_makes_the_next_collective_fail_not_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    rank, outcome, waited = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and outcome != "no error"
    assert waited < 60                                # bounded by the process-group timeout, not forever


def test_reference_arm_runs_the_oracle_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "3", "--warmup", "1"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                        "tiny", "--steps", "1", "--warmup", "1"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_prefill_slots_place_each_new_token_at_its_position():
    """Writing rows through bench.prefill_slots (oracle write) and gathering
    each sequence puts new token i at position n - q_len + i."""
    from oracle import attention as OA
    from oracle import cache_ops as OC

    w = syn.custom_prefill([37, 16, 5, 70], [20, 16, 1, 0], 2, 1, 4, "fp32", seed=3)
    tables = syn.placement_tables(w)
    slots = bench.prefill_slots(w, tables)
    rows = int(w.qlens.sum())
    assert len(slots) == rows and len(set(slots.tolist())) == rows
    kc = np.zeros((w.num_blocks, 1, 16, 4), np.int32)
    k_new = (np.arange(rows, dtype=np.int32) + 1)[:, None, None] * np.ones((1, 1, 4), np.int32)
    kc2, _ = OC.write_kv(k_new, k_new, slots, kc, kc)
    row = 0
    for s, (n, q) in enumerate(zip(w.lens, w.qlens)):
        K = OA.gather_sequence(kc2, tables[s], int(n), 0)
        for i in range(int(q)):
            assert K[int(n - q) + i, 0] == row + 1
            row += 1
        assert (K[: int(n - q)] == 0).all()           # the cached prefix is untouched


def test_prefill_flops_count_visible_pairs():
    w = syn.custom_prefill([10, 4], [3, 4], 8, 2, 64, "bf16")
    # sequence 0: rows at positions 7, 8, 9 see 8 + 9 + 10 keys; sequence 1: 1 + 2 + 3 + 4
    assert bench.prefill_flops(w.lens, w.qlens, w) == (27 + 10) * 8 * 4 * 64


def test_prefill_reference_arm_runs_the_oracle_on_cpu():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "prefill",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_chunked_workload_has_few_rows_over_long_prefixes():
    w = syn.workload("chunked")
    prefix = w.lens - w.qlens
    assert w.batch == 4 and w.n_q_heads == 32 and w.n_kv_heads == 8 and w.head_dim == 128
    assert ((prefix >= 16384) & (prefix <= 32768)).all() and ((w.qlens >= 64) & (w.qlens <= 256)).all()
    # the pool holds every sequence's pages, each physical block used at most once
    nblocks = int((-(-w.lens // w.block_size)).sum())
    assert w.num_blocks >= nblocks and len(set(w.placement[:nblocks].tolist())) == nblocks


class _FakeNvml:
    """Three GPUs known to NVML by index, UUID and PCI bus id."""

    devices = [("GPU-aaaa", "00000000:1B:00.0"), ("GPU-bbbb", "00000000:43:00.0"), ("GPU-cccc", "00000000:9C:00.0")]

    def __init__(self, uuid_ok=True):
        self.uuid_ok = uuid_ok

    def nvmlDeviceGetHandleByUUID(self, uuid):
        if not self.uuid_ok:
            raise RuntimeError("no UUID lookup")
        return next(i for i, (u, _) in enumerate(self.devices) if u == uuid)

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        return next(i for i, (_, b) in enumerate(self.devices) if b == bus)

    def nvmlDeviceGetHandleByIndex(self, i):
        return i


def test_clock_sampler_finds_the_cuda_device_not_the_nvml_index(monkeypatch):
    """CUDA device 0 of a process that sees only the third GPU is NVML device 2."""
    import types

    props = types.SimpleNamespace(uuid="cccc", pci_domain_id=0, pci_bus_id=0x9C, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda i: props)
    assert bench.nvml_handle(_FakeNvml(), 0) == (2, "uuid")
    assert bench.nvml_handle(_FakeNvml(uuid_ok=False), 0) == (2, "pci")

    def no_props(i):
        raise RuntimeError("no CUDA")

    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", no_props)
    assert bench.nvml_handle(_FakeNvml(), 0) == (0, "index")


def test_sweep_defaults_and_l2_note():
    a = bench.parse_args([])
    assert a.config == "gqa" and a.sweep == "auto" and a.sweep_steps >= 20 >= a.sweep_warmup
    assert set(bench.SWEEP) == {"mha7b", "long", "cow", "tiny", "prefill", "chunked"}
    assert all(c in bench.DESCRIPTIONS for c in bench.SWEEP)
    tiny = syn.workload("tiny")
    assert "stays in the 126 MB L2" in bench.l2_note(bench.algorithmic_bytes(tiny.lens, tiny))
    gqa = syn.workload("gqa")
    assert "far above the 126 MB L2" in bench.l2_note(bench.algorithmic_bytes(gqa.lens, gqa))
