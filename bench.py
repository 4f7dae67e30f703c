"""Benchmark of the paged KV-cache decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long|mha|gqa|prefix|tiny]
    python bench.py --kv fp8 ...              (the step on E4M3 pools: quantising write + decode)
    python bench.py --op multi --q-len n ...  (several query tokens per sequence)
    python bench.py --op copy_blocks ...      (copy-on-write block copies)
    python bench.py --config prefix --plain-decode ...  (the prefix batch without the shared-prefix path)
    python bench.py --impl reference ...      (the fp64 CPU oracle, timed on host cores)

The default workload is the long-context one (8 sequences of 32k-128k tokens,
64 query heads over 8 kv heads, 32-block partitions), the largest that fits one
GPU; --config picks another.

One step = one pass of the hot path over one batch: the cache write of each
sequence's newest token (pa_cache_write), then the decode (the block-table
walk with split-K partials, pa_decode_partitions, and the log-sum-exp merge,
pa_decode_reduce).  Inputs are resident in HBM; L2 is flushed before every
step (a 512 MiB write, then a 512 MiB read so no dirty lines or pending
write-backs are left for the next step), outside the timed events.  Times are CUDA events on the
launching stream; with N > 1 (torchrun) every rank runs its own replica of the
workload (seed + rank, no data exchange) and the step time is the max over
ranks.  Prints one JSON line.

metric: KV GB/s = algorithmic bytes of a step / step time, where the bytes are
the KV of every token attended (each distinct physical block counted once:
shared prefix blocks are read once), q, out, table entries and lengths, plus
the cache write's reads and writes.  Decode tokens/s = sequences / step time.

Besides value and the dominant kernel's roofline the line carries e2e (the
same steps through the public API from pinned host buffers, run as a serving
loop: the next step's inputs copied in and the previous step's result read
back while a step computes, every step's copies inside the timed region),
e2e_serial (copy in, compute, read back one after another, L2 flushed before
each step), warm_l2 for a batch that shares a prompt (the steps without the
flush), the oracle's cpu_baseline, NVML clocks and the launch count.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import itertools
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_432_b200 import workload as wl  # noqa: E402

FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
METRIC = "paged decode attention KV GB/s and decode tokens/s on 1 B200 vs 8 TB/s HBM roofline"


# ---------------------------------------------------------------- bytes accounting
def algorithmic_bytes(w: wl.Workload, kv_bytes=None) -> dict:
    """Bytes a step must move at minimum.  KV: every (distinct physical block,
    kv head) slice attended, counted once, with the valid slots only.
    kv_bytes: bytes per cached element (1 for E4M3 pools; default the
    workload's element size)."""
    e = w.elem_bytes
    ek = e if kv_bytes is None else kv_bytes
    D, Hkv, Hq = w.head_dim, w.num_kv_heads, w.num_q_heads
    valid = {}
    for L, t in zip(w.lens_host, w.tables_host):
        for j, b in enumerate(t):
            valid[b] = max(valid.get(b, 0), min(16, L - 16 * j))
    kv_unique = 2 * sum(valid.values()) * Hkv * D * ek
    kv_logical = 2 * sum(w.lens_host) * Hkv * D * ek
    n_blocks_read = sum(len(t) for t in w.tables_host)
    q_out = 2 * w.num_seqs * Hq * D * e
    meta = 4 * n_blocks_read + 4 * w.num_seqs
    decode = kv_unique + q_out + meta
    T = int(w.slot_mapping.numel())
    write = 2 * T * Hkv * D * (e + ek) + 8 * T  # new k, v read; their slots written
    return dict(decode=decode, write=write, step=decode + write, kv_unique=kv_unique,
                kv_logical=kv_logical, q_out=q_out, meta=meta)


def resolve_partition_blocks(pb: int) -> int:
    """The partition setting the decode runs with (as pa_decode_partition_blocks
    resolves it): > 0 fixed partitions, -1 never split (1 << 24), 0 balanced."""
    return pb if pb > 0 else ((1 << 24) if pb == -1 else 0)


def workload_config(w: wl.Workload, pb: int, kv: str = "bf16") -> dict:
    """The workload a line measures; both arms (the GPU path and the oracle)
    report the same dict for the same arguments."""
    by = algorithmic_bytes(w, kv_bytes=1 if kv == "fp8" else None)
    return {
        "workload": w.name,
        "desc": w.desc,
        "seed": w.seed,
        "num_seqs": w.num_seqs,
        "tokens": sum(w.lens_host),
        "max_seq_len": w.max_seq_len,
        "num_q_heads": w.num_q_heads,
        "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "pool_blocks": w.num_blocks,
        "partition_blocks": pb,
        "split": "balanced (equal blocks per warp)" if pb == 0 else (
            "never" if pb >= (1 << 24) else f"fixed {pb}-block partitions"),
        "new_tokens": int(w.slot_mapping.numel()),
        "shared_prefix_blocks": w.shared_prefix_blocks,
        "slot_utilisation": round(sum(w.lens_host) / (16 * sum(len(t) for t in w.tables_host)), 5),
        "kv": "e4m3 codes, per-head fp32 scales" if kv == "fp8" else (
            "bf16" if w.dtype == torch.bfloat16 else "f32"),
        "l2": f"inputs larger than L2 (distinct KV read per step {by['kv_unique'] / 1e6:.0f} MB vs 126 MB "
              "of L2) and L2 flushed before every GPU step (512 MiB write + 512 MiB read, outside "
              "the timed events)",
    }


# the device sources of the decode kernel (decode_bf16_mma_kernel, bf16 and
# E4M3): a committed traffic figure counts only while these are unchanged
DECODE_SOURCES = ("common.cuh", "items.cuh", "decode_mma.cuh")


def source_digest(files=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    for name in files:
        h.update(open(os.path.join(ROOT, "paged_kv_cache_432_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def load_peaks() -> tuple:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_tensor_peak() -> tuple:
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure (a kernel
    timed alone), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def causal_flops(lens, n_per_seq, num_q_heads, head_dim) -> int:
    """Algorithmic FLOPs of several query tokens per sequence: token k of n
    sees L - n + k + 1 keys; per (token, head, key) 2 D for q . k and 2 D for
    p . v."""
    tot = 0
    for L, n in zip(lens, n_per_seq):
        n = min(n, L)
        tot += n * (L - n) + n * (n + 1) // 2
    return 4 * head_dim * num_q_heads * tot


def load_traffic(tag: str):
    """dram bytes per launch of the decode kernel from a committed ncu summary
    (profiles/<tag>.json), if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", f"{tag}.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None
    if d.get("source_digest") != source_digest():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks (NVML)
_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}
_BAD = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    def __init__(self, device: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.err = None
        self.h = None
        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
            ident = vis[device].strip() if vis and vis[0] != "" and device < len(vis) else str(device)
            if ident.startswith("GPU-") or ident.startswith("MIG-"):
                self.h = pynvml.nvmlDeviceGetHandleByUUID(ident)
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(int(ident))
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.err = f"nvml unavailable: {e}"
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self.t.join()

    def summary(self) -> dict:
        if self.h is None or not self.samples:
            return {"error": self.err or "no samples"}
        names = sorted(v for k, v in _REASONS.items() if self.reasons & k and v != "gpu_idle")
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "source": "nvml, 5 ms period"}


# ---------------------------------------------------------------- distributed plumbing
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def _reduce(x: float, ws: int, op: str, device) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(step_ms: float, step_bytes: float, seqs: int, ws: int, device="cuda") -> dict:
    """Whole-job numbers of a weak-scaling run: every rank processed its own
    replica; the job took as long as the slowest rank."""
    t = _reduce(step_ms, ws, "max", device)
    b = _reduce(float(step_bytes), ws, "sum", device)
    n = _reduce(float(seqs), ws, "sum", device)
    return {"step_ms": t, "bytes": b, "seqs": n, "gbs": b / (t * 1e-3) / 1e9,
            "tokens_per_s": n / (t * 1e-3)}


def max_over_ranks(x: float, ws: int, device="cuda") -> float:
    return _reduce(x, ws, "max", device)


def replica_seed(base: int, rank: int) -> int:
    """Each rank draws its own replica of the workload."""
    return base + rank


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------- CPU oracle timing
def oracle_step_sample(w: wl.Workload, h: dict, seqs: list) -> tuple:
    """Runs the oracle (cache write + decode) for the given sequences; returns
    (seconds, algorithmic bytes of that sample)."""
    import numpy as np

    import oracle

    sel = np.array(seqs)
    rows = [(s, qh) for s in seqs for qh in range(w.num_q_heads)]
    t0 = time.perf_counter()
    oracle.cache_write(h["nk"][sel], h["nv"][sel], h["sm"][sel], h["kc"], h["vc"], inplace=True)
    oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, rows=rows)
    return time.perf_counter() - t0, sample_bytes(w, seqs)


def sample_bytes(w: wl.Workload, seqs: list) -> int:
    """Algorithmic bytes of the step restricted to the given sequences: their
    KV once per kv head, q and out, their table entries, the cache write."""
    e, D, Hkv, Hq = w.elem_bytes, w.head_dim, w.num_kv_heads, w.num_q_heads
    kv = 2 * sum(w.lens_host[s] for s in seqs) * Hkv * D * e
    return kv + 2 * len(seqs) * Hq * D * e + 4 * sum(len(w.tables_host[s]) for s in seqs) + \
        2 * (2 * len(seqs) * Hkv * D * e)


def host_arrays(w: wl.Workload) -> dict:
    return dict(q=wl.as_numpy(w.q), kc=wl.as_numpy(w.k_cache), vc=wl.as_numpy(w.v_cache),
                bt=wl.as_numpy(w.block_tables), sl=wl.as_numpy(w.seq_lens),
                nk=wl.as_numpy(w.new_k), nv=wl.as_numpy(w.new_v), sm=wl.as_numpy(w.slot_mapping))


def cpu_baseline(w: wl.Workload, budget_s: float = 20.0) -> dict:
    """The oracle as it stands, single-threaded, on a bounded sample: whole
    sequences (all heads) in order until about budget_s of work."""
    h = host_arrays(w)
    total_t, total_b, seqs = 0.0, 0, []
    s = 0
    while s < w.num_seqs and total_t < budget_s:
        dt, by = oracle_step_sample(w, h, [s])
        total_t += dt
        total_b += by
        seqs.append(s)
        s += 1
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{len(seqs)} of {w.num_seqs} sequences (all {w.num_q_heads} q heads, cache "
                      f"write + decode), {total_t:.1f} s single-threaded fp64",
            "tokens_per_s": round(len(seqs) / total_t, 3),
            "all_cores": cpu_baseline_all_cores(w, h, seqs, budget_s / 2)}


def cpu_baseline_all_cores(w: wl.Workload, h: dict, seqs: list, budget_s: float) -> dict:
    """The same oracle work on the same sequences, spread over every host core
    this process may use (the C oracle runs without the interpreter lock):
    the sample's cache writes, then decode tasks of whole kv heads of one
    sequence, about four per core (fewer, larger tasks keep the interpreter's
    share small), longest first.  Whole passes are repeated until about
    budget_s of wall time."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle

    cores = len(os.sched_getaffinity(0))
    g, Hkv = w.num_q_heads // w.num_kv_heads, w.num_kv_heads
    chunks = min(Hkv, -(-4 * cores // len(seqs)))  # kv-head chunks per sequence
    bounds = [Hkv * c // chunks for c in range(chunks + 1)]
    tasks = [(s, bounds[c], bounds[c + 1]) for s in sorted(seqs, key=lambda s: -w.lens_host[s])
             for c in range(chunks)]

    def write(s):
        sel = np.array([s])
        oracle.cache_write(h["nk"][sel], h["nv"][sel], h["sm"][sel], h["kc"], h["vc"], inplace=True)

    def decode(task):
        s, k0, k1 = task
        oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale,
                            rows=[(s, qh) for qh in range(k0 * g, k1 * g)])

    per_pass = sample_bytes(w, seqs)
    passes, t0 = 0, time.perf_counter()
    with ThreadPoolExecutor(max_workers=cores) as ex:
        while True:
            list(ex.map(write, seqs))
            list(ex.map(decode, tasks))
            passes += 1
            if time.perf_counter() - t0 >= budget_s:
                break
    wall = time.perf_counter() - t0
    return {"value": round(passes * per_pass / wall / 1e9, 4), "unit": "GB/s", "cores": cores,
            "sample": f"the same {len(seqs)} sequences, {passes} pass(es) of {len(tasks)} "
                      f"decode tasks, {wall:.1f} s wall on {cores} threads"}


def oracle_unit_sample(w: wl.Workload, h: dict, units: list) -> tuple:
    """Runs the oracle on (sequence, kv head) units: the cache write of each
    touched sequence's newest token (all heads), then the decode of every
    query head of each unit.  Returns (seconds, algorithmic bytes)."""
    import numpy as np

    import oracle

    g = w.num_q_heads // w.num_kv_heads
    seqs = sorted({s for s, _ in units})
    sel = np.array(seqs)
    rows = [(s, kh * g + i) for s, kh in units for i in range(g)]
    t0 = time.perf_counter()
    oracle.cache_write(h["nk"][sel], h["nv"][sel], h["sm"][sel], h["kc"], h["vc"], inplace=True)
    oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, rows=rows)
    dt = time.perf_counter() - t0
    e, D = w.elem_bytes, w.head_dim
    by = sum(2 * w.lens_host[s] * D * e + 2 * g * D * e + 4 * len(w.tables_host[s]) for s, _ in units)
    by += len(seqs) * 2 * (2 * w.num_kv_heads * D * e)
    return dt, by


def run_reference(args) -> None:
    """The reference arm: the fp64 oracle on host cores, on the same workload
    and metric as the GPU arm.  Each step is a bounded sample of the batch:
    a fixed number of (sequence, kv head) units, rotating over the batch,
    sized from one calibration unit so that warm-up and timed steps together
    take about --ref-budget-s seconds."""
    ws, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    ng = getattr(args, "prompt_groups", 1)
    extra = {"prompt_groups": ng} if ng > 1 else {}
    w = wl.make(args.config, seed=args.seed, device="cpu", max_seqs=args.max_seqs, **extra)
    h = host_arrays(w)
    Hkv = w.num_kv_heads
    all_units = [(s, kh) for s in range(w.num_seqs) if w.lens_host[s] > 0 for kh in range(Hkv)]
    t_unit, _ = oracle_unit_sample(w, h, [max(all_units, key=lambda u: w.lens_host[u[0]])])
    per_step = max(1, int(args.ref_budget_s / (args.warmup + args.steps) / max(t_unit, 1e-6)))
    per_step = min(per_step, len(all_units))
    times, nbytes, nunits = [], [], []
    cur = 0
    for i in range(args.warmup + args.steps):
        units = [all_units[(cur + k) % len(all_units)] for k in range(per_step)]
        cur = (cur + per_step) % len(all_units)
        dt, by = oracle_unit_sample(w, h, units)
        if i >= args.warmup:
            times.append(dt)
            nbytes.append(by)
            nunits.append(len(units))
    T = sum(times)
    value = sum(nbytes) / T / 1e9
    sample = (f"{per_step} (sequence, kv head) unit(s) per step (each: all {w.num_q_heads // Hkv} query "
              f"heads of the unit, plus the cache write of its sequence's new token), rotating over "
              f"the batch's {len(all_units)} units; single-threaded fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * T / len(times), 3),
        "step_ms": {"mean": round(1e3 * T / len(times), 3), "median": round(1e3 * statistics.median(times), 3),
                    "min": round(1e3 * min(times), 3)},
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, resolve_partition_blocks(w.partition_blocks if args.partition_blocks is None
                                                              else args.partition_blocks), args.kv),
        "tokens_per_s": round(sum(nunits) / Hkv / T, 3),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args) -> None:
    from paged_kv_cache_432_b200 import build as pa_build
    from paged_kv_cache_432_b200 import pagedattn as pa

    ws, rank, local = dist_setup()
    if rank == 0:
        pa_build.build()
    barrier(ws)
    dev = torch.device("cuda", local)
    extra = {"prompt_groups": args.prompt_groups} if args.prompt_groups > 1 else {}
    w = wl.make(args.config, seed=replica_seed(args.seed, rank), device=dev, max_seqs=args.max_seqs, **extra)
    pb = w.partition_blocks if args.partition_blocks is None else args.partition_blocks
    msl = w.max_seq_len
    resolved_pb = pa.partition_blocks(w.num_seqs, w.num_kv_heads, msl, pb)
    fp8 = args.kv == "fp8"
    if fp8:  # E4M3 pools with the workload's structure, per-head scales
        if w.dtype != torch.bfloat16:
            raise SystemExit("--kv fp8 needs a bf16 workload")
        w.k_cache, w.v_cache, k_scale, v_scale = wl.fp8_pools(w)
        k_inv, v_inv = (1.0 / k_scale).float(), (1.0 / v_scale).float()
        torch.cuda.empty_cache()
    # a batch sharing a prompt prefix goes through the shared-prefix decode
    # (several prompts: the prompt-group form)
    groups = len(w.group_blocks_host) > 1 and max(w.group_blocks_host) > 0
    use_sp = (w.shared_prefix_blocks > 0 or groups) and not args.plain_decode and not fp8
    maxs = max(w.group_blocks_host) if groups else 0
    if use_sp and groups:
        n = pa.shared_prefix_groups_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, msl,
                                                   maxs, len(w.group_blocks_host), pb)
        wsp = torch.empty(n, dtype=torch.uint8, device=dev)
    elif use_sp:
        n = pa.shared_prefix_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, msl,
                                            w.shared_prefix_blocks, pb)
        wsp = torch.empty(n, dtype=torch.uint8, device=dev)
    else:
        wsp = pa.alloc_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, msl, pb, device=dev)
    split = wsp is not None
    out = torch.empty_like(w.q)
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        # evict everything: write a buffer 4x the L2, then read another 4x the
        # L2 so the lines left behind are clean and the write-backs of the
        # written lines have drained (none lands in the next timed step)
        flush_w.zero_()
        flush_r.view(torch.float32).sum()  # a read-only reduction (no dtype-converting copy)
    stream = torch.cuda.current_stream(dev)
    by = algorithmic_bytes(w, kv_bytes=1 if fp8 else None)
    chunks = math.ceil(w.num_seqs / 2048)
    launches_per_step = 1 + chunks + (chunks if split else 0) + (1 if use_sp else 0)

    def shared_prefix_call(q, block_tables, seq_lens, o=None):
        o = out if o is None else o
        if groups:
            pa.decode_shared_prefix_groups(q, w.k_cache, w.v_cache, block_tables, seq_lens, w.scale, w.group_start,
                                           w.group_blocks, maxs, out=o, max_seq_len=msl, partition_blocks=pb,
                                           workspace=wsp, stream=stream)
        else:
            pa.decode_shared_prefix(q, w.k_cache, w.v_cache, block_tables, seq_lens, w.scale,
                                    w.shared_prefix_blocks, out=o, max_seq_len=msl, partition_blocks=pb,
                                    workspace=wsp, stream=stream)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if fp8:  # quantising write, then the E4M3 decode kernel and its merge
            pa.cache_write_fp8(w.new_k, w.new_v, w.slot_mapping, w.k_cache, w.v_cache, k_inv, v_inv, stream)
            if ev is not None:
                ev[1].record(stream)
            pa.decode_fp8_partitions(w.q, w.k_cache, w.v_cache, k_scale, v_scale, w.block_tables, w.seq_lens,
                                     w.scale, out, msl, pb, wsp, stream)
            if ev is not None:
                ev[2].record(stream)
            if split:
                pa.decode_fp8_reduce(w.seq_lens, out, w.num_kv_heads, w.max_blocks_per_seq, msl, pb, wsp, stream)
            if ev is not None:
                ev[3].record(stream)
            return
        pa.cache_write(w.new_k, w.new_v, w.slot_mapping, w.k_cache, w.v_cache, stream)
        if ev is not None:
            ev[1].record(stream)
        if use_sp:  # prefix kernel + private-part decode + merge, one call
            shared_prefix_call(w.q, w.block_tables, w.seq_lens)
            if ev is not None:
                ev[2].record(stream)
                ev[3].record(stream)
            return
        pa.decode_partitions(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, out, msl,
                             pb, wsp, stream)
        if ev is not None:
            ev[2].record(stream)
        if split:
            pa.decode_reduce(w.seq_lens, out, w.num_kv_heads, w.max_blocks_per_seq, msl, pb, wsp, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)
    if pa.device_error() != 0:
        raise RuntimeError("device error flagged during warm-up")

    def timed():
        """Two timed loops over the same steps: (a) events at step boundaries
        only, so consecutive kernels overlap as they do in use (programmatic
        dependent launch) -> the step time; (b) events between the kernels ->
        each kernel's own duration (the roofline's)."""
        K = args.steps
        ev_step = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        ev_k = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        barrier(ws)
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as cs:
            for k in range(K):
                flush_l2()
                ev_step[k][0].record(stream)
                step()
                ev_step[k][1].record(stream)
            torch.cuda.synchronize(dev)
            for k in range(K):
                flush_l2()
                step(ev_k[k])
            torch.cuda.synchronize(dev)
        barrier(ws)
        per_step = [a.elapsed_time(b) for a, b in ev_step]
        dec = sum(e[1].elapsed_time(e[2]) for e in ev_k)
        red = sum(e[2].elapsed_time(e[3]) for e in ev_k)
        wr = sum(e[0].elapsed_time(e[1]) for e in ev_k)
        return per_step, dec, red, wr, cs.summary()

    per_step, dec, red, wr, clocks = timed()
    if set(clocks.get("reasons", [])) & _BAD:  # re-measure once
        per_step, dec, red, wr, clocks = timed()
        clocks["remeasured"] = True
    K = args.steps
    tot = sum(per_step)
    step_stats = {"mean": round(max_over_ranks(tot / K, ws), 5),
                  "median": round(max_over_ranks(statistics.median(per_step), ws), 5),
                  "min": round(max_over_ranks(min(per_step), ws), 5),
                  "how": "CUDA events at step boundaries; each statistic is the max over ranks"}
    agg = aggregate(tot / K, by["step"], w.num_seqs, ws)
    step_ms, total_bytes, total_seqs, value = agg["step_ms"], agg["bytes"], agg["seqs"], agg["gbs"]
    dec_ms = max_over_ranks(dec / K, ws)
    red_ms = max_over_ranks(red / K, ws)
    wr_ms = max_over_ranks(wr / K, ws)

    # ---- a batch sharing a prompt also reports a warm-L2 step: no flush
    # between steps, so the shared blocks stay in L2 from one step to the next
    warm = None
    if w.shared_prefix_blocks > 0 or groups:
        n_w = max(3, min(K, 50))
        for _ in range(2):
            step()
        evw = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_w)]
        barrier(ws)
        torch.cuda.synchronize(dev)
        for k in range(n_w):
            evw[k][0].record(stream)
            step()
            evw[k][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(ws)
        w_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evw) / n_w, ws)
        warm = {"ms_per_step": round(w_ms, 5), "value": round(total_bytes / (w_ms * 1e-3) / 1e9, 2),
                "unit": "GB/s", "steps": n_w,
                "how": "the same steps with no L2 flush between them (events at step boundaries)"}

    # ---- end to end through the public API: inputs from pinned host memory,
    # result read back, every step
    e2e, e2e_serial = None, None
    if not args.no_e2e:
        # a step's inputs travel in one pinned staging buffer (one H2D copy),
        # each at a 256-byte aligned offset; the device tensors are views.  Two
        # slots (inputs and output), so that copies of one step can overlap
        # the compute of another.
        names = ["q", "new_k", "new_v", "slot_mapping", "block_tables", "seq_lens"]
        src = {n: getattr(w, n).contiguous() for n in names}
        offs, off = {}, 0
        for n in names:
            offs[n] = off
            off += (src[n].numel() * src[n].element_size() + 255) // 256 * 256

        def make_slot():
            hb = torch.empty(off, dtype=torch.uint8, pin_memory=True)
            db = torch.empty(off, dtype=torch.uint8, device=dev)
            di = {}
            for n in names:
                nb = src[n].numel() * src[n].element_size()
                hb[offs[n]:offs[n] + nb].copy_(src[n].view(-1).view(torch.uint8).cpu())
                di[n] = db[offs[n]:offs[n] + nb].view(src[n].dtype).view(src[n].shape)
            return {"hb": hb, "db": db, "di": di, "o": torch.empty_like(out),
                    "ho": torch.empty(out.shape, dtype=out.dtype, pin_memory=True)}

        slots = [make_slot(), make_slot()]
        h2d = sum(src[n].numel() * src[n].element_size() for n in names)
        d2h = slots[0]["ho"].numel() * slots[0]["ho"].element_size()

        def compute(sl):
            """The step through the public API from slot sl's device inputs into its output."""
            di, o = sl["di"], sl["o"]
            if fp8:
                pa.cache_write_fp8(di["new_k"], di["new_v"], di["slot_mapping"], w.k_cache, w.v_cache,
                                   k_inv, v_inv, stream)
                pa.decode_fp8(di["q"], w.k_cache, w.v_cache, k_scale, v_scale, di["block_tables"],
                              di["seq_lens"], w.scale, out=o, max_seq_len=msl, partition_blocks=pb,
                              workspace=wsp, stream=stream)
                return
            pa.cache_write(di["new_k"], di["new_v"], di["slot_mapping"], w.k_cache, w.v_cache, stream)
            if use_sp:
                shared_prefix_call(di["q"], di["block_tables"], di["seq_lens"], o)
            else:
                pa.decode(di["q"], w.k_cache, w.v_cache, di["block_tables"], di["seq_lens"], w.scale,
                          out=o, max_seq_len=msl, partition_blocks=pb, workspace=wsp, stream=stream)

        def serial_step():  # copy in, compute, read back, one after another
            sl = slots[0]
            sl["db"].copy_(sl["hb"], non_blocking=True)
            compute(sl)
            sl["ho"].copy_(sl["o"], non_blocking=True)

        copy_in = torch.cuda.Stream(device=dev)
        copy_out = torch.cuda.Stream(device=dev)

        def pipelined(n):
            """n steps as a serving loop runs them: step k+1's inputs are copied
            in (copy_in) and step k-1's result read back (copy_out) while step
            k computes; events keep each slot's inputs until its compute ends
            and its output until it was read back.  Returns ms per step, from
            before the first step's copy-in to after the last step's read-back."""
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_c = [torch.cuda.Event() for _ in range(n)]
            ev_o = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            copy_in.wait_event(t0)

            def copy_step_in(k):
                sl = slots[k % 2]
                if k >= 2:
                    copy_in.wait_event(ev_c[k - 2])  # the slot's inputs are free once step k-2 computed
                with torch.cuda.stream(copy_in):
                    sl["db"].copy_(sl["hb"], non_blocking=True)
                ev_in[k].record(copy_in)

            copy_step_in(0)
            for k in range(n):
                if k + 1 < n:
                    copy_step_in(k + 1)
                sl = slots[k % 2]
                stream.wait_event(ev_in[k])
                if k >= 2:
                    stream.wait_event(ev_o[k - 2])  # the slot's output was read back
                compute(sl)
                ev_c[k].record(stream)
                copy_out.wait_event(ev_c[k])
                with torch.cuda.stream(copy_out):
                    sl["ho"].copy_(sl["o"], non_blocking=True)
                ev_o[k].record(copy_out)
            stream.wait_event(ev_o[n - 1])
            t1.record(stream)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1) / n

        n_e2e = max(3, min(K, 50))
        # pipelined: the headline end-to-end figure
        pipelined(max(2, args.warmup))
        barrier(ws)
        torch.cuda.synchronize(dev)
        p_ms = max_over_ranks(pipelined(n_e2e), ws)
        barrier(ws)
        e2e = {"value": round(total_bytes / (p_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(p_ms, 4),
               "steps": n_e2e,
               "how": ("pa_cache_write + the decode entry point from device copies of pinned host inputs, result "
                       "read back to pinned host memory, every step; two slots: the next step's copy-in and the "
                       "previous step's read-back overlap the current step's compute; one event pair around all "
                       "steps; L2 not flushed between steps (the KV read per step exceeds L2" +
                       ("; a shared prompt's blocks stay in L2 from step to step, as in serving)"
                        if (w.shared_prefix_blocks > 0 or groups) else ")"))}
        # serial: copy in, compute, read back, L2 flushed before each step (outside the events)
        for _ in range(args.warmup):
            flush_l2()
            serial_step()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_e2e)]
        barrier(ws)
        torch.cuda.synchronize(dev)
        for k in range(n_e2e):
            flush_l2()
            evs[k][0].record(stream)
            serial_step()
            evs[k][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(ws)
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / n_e2e, ws)
        e2e_serial = {"value": round(total_bytes / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                      "ms_per_step": round(e_ms, 4), "steps": n_e2e,
                      "how": "copy in, compute, read back on one stream, L2 flushed before each step"}

    if pa.device_error() != 0:
        raise RuntimeError("device error flagged during timing")

    peak, peak_kind = load_peaks()
    achieved = by["decode"] / (dec_ms * 1e-3) / 1e9
    kname = "decode_bf16_mma_kernel" if w.dtype == torch.bfloat16 else "decode_f32_simt_kernel"
    if use_sp:
        kname = ("pa_decode_shared_prefix_groups" if groups else "pa_decode_shared_prefix") + \
            " (attn_tiles_tc_kernel + decode_bf16_mma_kernel + reduce, timed together)"
    if fp8:
        kname = "decode_bf16_mma_kernel, E4M3 form (pa_decode_fp8_partitions; the merge timed apart)"
    roof = {"bound": "hbm", "kernel": kname, "achieved": round(achieved, 1), "peak": peak,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6650 GB/s", "unit": "GB/s", "frac": round(achieved / peak, 4),
            "frac_of_8TBs": round(achieved / 8000.0, 4),
            "algorithmic_bytes_per_launch": by["decode"],
            "traffic": load_traffic(f"decode_{'fp8' if fp8 else 'bf16'}_mma_{w.name}")}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not fp8:
        cpu = cpu_baseline(w, budget_s=args.cpu_budget_s)

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "step_ms": step_stats,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e4m3 KV, f16 MMA" if fp8 else "bf16") if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": workload_config(w, resolved_pb, args.kv),
        "tokens_per_s": round(total_seqs / (step_ms * 1e-3), 1),
        "kernel_ms": {"cache_write": round(wr_ms, 5), "decode_partitions": round(dec_ms, 5),
                      "lse_reduce": round(red_ms, 5),
                      "how": "CUDA events between the kernels, in a second timed loop of the same steps"},
        "bytes_per_step": by,
        "roofline": roof,
        "e2e": e2e,
        "e2e_serial": e2e_serial,
        "warm_l2": warm,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": launches_per_step * K,
        "gpu_launches_note": "per timed loop: cache write, decode, reduce per step",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_copy_blocks(args) -> None:
    """Copy-on-write block copies (pa_copy_blocks) on the workload's pool: 2048
    pairs of distinct random blocks per step, L2 flushed between steps."""
    from paged_kv_cache_432_b200 import build as pa_build
    from paged_kv_cache_432_b200 import pagedattn as pa

    ws, rank, local = dist_setup()
    if rank == 0:
        pa_build.build()
    barrier(ws)
    dev = torch.device("cuda", local)
    w = wl.make(args.config, seed=replica_seed(args.seed, rank), device=dev)
    n = min(2048, w.num_blocks // 2)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(args.seed + rank))
    src = perm[:n].to(torch.int32).to(dev)
    dst = perm[n:2 * n].to(torch.int32).to(dev)
    block_bytes = w.k_cache[0].numel() * w.elem_bytes
    moved = 2 * 2 * n * block_bytes  # both pools, read + write
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        pa.copy_blocks(w.k_cache, w.v_cache, src, dst, stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as cs:
        for e in evs:
            flush_w.zero_()
            flush_r.view(torch.float32).sum()
            e[0].record(stream)
            pa.copy_blocks(w.k_cache, w.v_cache, src, dst, stream)
            e[1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    agg = aggregate(sum(a.elapsed_time(b) for a, b in evs) / args.steps, moved, n, ws)
    peak, peak_kind = load_peaks()
    if pa.device_error() != 0:
        raise RuntimeError("device error flagged")
    line = {"metric": "copy-on-write block copy GB/s (read + write)", "value": round(agg["gbs"], 1),
            "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(agg["step_ms"], 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": {"workload": w.name, "op": "pa_copy_blocks", "pairs": n, "block_bytes_per_pool": block_bytes,
                       "l2": "flushed before every step (512 MiB write + 512 MiB read)"},
            "roofline": {"bound": "hbm", "kernel": "copy_blocks_kernel", "achieved": round(agg["gbs"] / ws, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(agg["gbs"] / ws / peak, 4),
                         "peak_source": peak_kind, "traffic": None},
            "clocks": cs.summary(), "gpu_launches": args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_multi(args) -> None:
    """Several query tokens per sequence (pa_decode_multi): the check step of
    speculative decoding with q_len - 1 drafted tokens, or (group x q_len > 16)
    a prefill chunk of q_len tokens on the tensor-memory tile kernel.  A
    sequence shorter than q_len takes all its positions as query tokens.  The
    KV of every sequence is read once for all its query tokens (per tile)."""
    from paged_kv_cache_432_b200 import build as pa_build
    from paged_kv_cache_432_b200 import pagedattn as pa

    ws, rank, local = dist_setup()
    if rank == 0:
        pa_build.build()
    barrier(ws)
    dev = torch.device("cuda", local)
    w = wl.make(args.config, seed=replica_seed(args.seed, rank), device=dev, max_seqs=args.max_seqs)
    nq = args.q_len
    n_per = [min(nq, L) for L in w.lens_host]
    gen = torch.Generator(device=dev).manual_seed(args.seed + 7)
    q = torch.randn((sum(n_per), w.num_q_heads, w.head_dim), generator=gen, device=dev).to(w.dtype)
    qs = torch.tensor([0] + list(itertools.accumulate(n_per)), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    pb = w.partition_blocks if args.partition_blocks is None else args.partition_blocks
    msl = w.max_seq_len
    n = pa.multi_workspace_size(w.num_seqs, q.shape[0], w.num_q_heads, w.num_kv_heads, w.head_dim, msl, pb)
    wsp = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    by = algorithmic_bytes(w)
    step_bytes = by["kv_unique"] + by["meta"] + 2 * q.numel() * w.elem_bytes
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, nq, out=out,
                        max_seq_len=msl, partition_blocks=pb, workspace=wsp, stream=stream)

    for _ in range(args.warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as cs:
        for e in evs:
            flush_w.zero_()
            flush_r.view(torch.float32).sum()
            e[0].record(stream)
            step()
            e[1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    step_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    agg = aggregate(step_ms, step_bytes, sum(n_per), ws)
    peak, peak_kind = load_peaks()
    if pa.device_error() != 0:
        raise RuntimeError("device error flagged")
    tiles = w.group * nq > 16  # more rows per (sequence, kv head) than one warp-level MMA holds
    flops = causal_flops(w.lens_host, n_per, w.num_q_heads, w.head_dim)
    if tiles:  # a prefill chunk: tensor-core bound
        tpeak, tkind = load_tensor_peak()
        ach = flops / (max_over_ranks(step_ms, ws) * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "attn_tiles_tc_kernel (+ merge when the keys are cut)",
                "achieved": round(ach, 1), "peak": tpeak, "unit": "TFLOP/s", "frac": round(ach / tpeak, 4),
                "peak_source": f"{tkind} (MEASURED_PEAKS.json bf16_tflops, burst)" if tkind == "measured"
                else "fallback 1590 TFLOP/s", "algorithmic_flops_per_step": flops, "traffic": None}
    else:
        roof = {"bound": "hbm", "kernel": "decode_bf16_mma_kernel + reduce", "achieved": round(agg["gbs"] / ws, 1),
                "peak": peak, "unit": "GB/s", "frac": round(agg["gbs"] / ws / peak, 4),
                "peak_source": peak_kind, "traffic": None}
    line = {"metric": f"multi-token paged decode KV GB/s ({nq} query tokens per sequence)",
            "value": round(agg["gbs"], 1), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(agg["step_ms"], 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w, pa.partition_blocks(w.num_seqs, w.num_kv_heads, msl, pb)),
                           op="pa_decode_multi", q_len=nq),
            "query_tokens_per_s": round(agg["tokens_per_s"], 1),
            "tflops": round(flops * ws / (agg["step_ms"] * 1e-3) / 1e12, 2),
            "roofline": roof,
            "clocks": cs.summary(), "gpu_launches": 2 * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="long", choices=list(wl.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="step", choices=["step", "copy_blocks", "multi"],
                    help="step: cache write + decode (the headline); copy_blocks: copy-on-write copies; "
                         "multi: several query tokens per sequence")
    ap.add_argument("--q-len", type=int, default=4, help="query tokens per sequence for --op multi")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="KV pool element type for --op step (fp8: E4M3 codes with per-head scales)")
    ap.add_argument("--partition-blocks", type=int, default=None)
    ap.add_argument("--prompt-groups", type=int, default=1,
                    help="--config prefix: that many prompts, each shared by a consecutive share of the batch")
    ap.add_argument("--max-seqs", type=int, default=None,
                    help="keep only the first N sequences of the workload (a smaller case of the same "
                         "shape, for profiler captures; not a bench line)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--plain-decode", action="store_true",
                    help="decode a shared-prefix batch with pa_decode instead of pa_decode_shared_prefix")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="--impl reference: host seconds the warm-up and timed steps take together")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.op == "copy_blocks":
        run_copy_blocks(args)
    elif args.op == "multi":
        run_multi(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
