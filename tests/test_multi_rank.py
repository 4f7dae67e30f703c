"""The N > 1 path of the benchmark, on CPU with the gloo backend (world size 2).

The decode work shards with no exchange: every rank runs its own replica of
the workload (weak scaling).  The only collectives are for measurement: the max
of the step time over ranks and the sums of bytes and sequences."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from paged_kv_cache_432_b200 import workload as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # each rank: its own replica, a different step time
        seed = bench.replica_seed(0, rank)
        p = wl.config_plan("gqa", seed=seed)
        step_ms = 1.0 + rank
        step_bytes = 1000.0 * (rank + 1)
        agg = bench.aggregate(step_ms, step_bytes, len(p.lens), ws, device="cpu")
        m = bench.max_over_ranks(0.5 * (rank + 1), ws, device="cpu")
        bench.barrier(ws)
        q.put((rank, agg, m, p.lens[:5]))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, agg, m, _ in res:
        assert agg["step_ms"] == 2.0            # the slowest rank
        assert agg["bytes"] == 3000.0           # both replicas' work
        assert agg["seqs"] == 512
        assert agg["gbs"] == pytest.approx(3000.0 / 2e-3 / 1e9)
        assert m == 1.0
    assert res[0][3] != res[1][3], "ranks must draw different replicas"


def test_single_rank_aggregation_is_identity():
    agg = bench.aggregate(2.5, 1e9, 64, 1)
    assert agg["step_ms"] == 2.5 and agg["bytes"] == 1e9 and agg["seqs"] == 64
    assert agg["gbs"] == pytest.approx(400.0)


def test_algorithmic_bytes_count_shared_prefix_once():
    w = wl.build([4096 + 10, 4096 + 20], 4, 2, 64, torch.bfloat16, seed=0, prefix_len=4096)
    by = bench.algorithmic_bytes(w)
    e, D, Hkv = 2, 64, 2
    assert by["kv_unique"] == 2 * (4096 + 10 + 20) * Hkv * D * e
    assert by["kv_logical"] == 2 * (2 * 4096 + 30) * Hkv * D * e
    assert by["decode"] == by["kv_unique"] + by["q_out"] + by["meta"]
