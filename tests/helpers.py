"""Shared test helpers: run the CUDA path and the oracle on the same seeded
inputs and compare them with the stated tolerances."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from paged_kv_cache_432_b200 import pagedattn as pa
from paged_kv_cache_432_b200 import workload as wl

# bf16 inputs: max-abs 2e-2 and normwise max-rel (max|g-o| / max|o|) 1e-2 of the
# fp64 oracle; fp32 inputs: max-abs 1e-5.
BF16_ABS, BF16_REL, F32_ABS = 2e-2, 1e-2, 1e-5


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close(gpu: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    mag = float(np.max(np.abs(ref))) if ref.size else 0.0
    if dtype == torch.bfloat16:
        assert err <= BF16_ABS, f"{what}: max_abs {err:.3e} > {BF16_ABS}"
        assert err <= BF16_REL * mag + 1e-30, f"{what}: normwise rel {err / max(mag, 1e-30):.3e} > {BF16_REL}"
    else:
        assert err <= F32_ABS, f"{what}: max_abs {err:.3e} > {F32_ABS}"
    return err, mag


def host(w: wl.Workload) -> dict:
    return dict(q=wl.as_numpy(w.q), kc=wl.as_numpy(w.k_cache), vc=wl.as_numpy(w.v_cache),
                bt=wl.as_numpy(w.block_tables), sl=wl.as_numpy(w.seq_lens),
                nk=wl.as_numpy(w.new_k), nv=wl.as_numpy(w.new_v), sm=wl.as_numpy(w.slot_mapping))


def gpu_decode(w: wl.Workload, partition_blocks=None, max_seq_len=None, q=None, k_cache=None,
               v_cache=None, block_tables=None):
    pb = w.partition_blocks if partition_blocks is None else partition_blocks
    msl = w.max_seq_len if max_seq_len is None else max_seq_len
    out = pa.decode(w.q if q is None else q, w.k_cache if k_cache is None else k_cache,
                    w.v_cache if v_cache is None else v_cache,
                    w.block_tables if block_tables is None else block_tables, w.seq_lens, w.scale,
                    max_seq_len=msl, partition_blocks=pb)
    torch.cuda.synchronize()
    return out


def oracle_decode(w: wl.Workload, h=None, rows=None):
    h = h or host(w)
    return oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, rows=rows)


def host_threads() -> int:
    return len(os.sched_getaffinity(0))


def oracle_decode_all_rows(w: wl.Workload, h=None) -> np.ndarray:
    """Every (sequence, query head) row of the oracle's decode, [N, Hq, D].
    The same plain oracle as oracle_decode, run as one task per (sequence, kv
    head) on host threads (the C oracle releases the interpreter lock), longest
    sequences first, so that full-size batches are compared in seconds."""
    h = h or host(w)
    N, Hq, D = h["q"].shape
    Hkv = h["kc"].shape[1]
    g = Hq // Hkv
    out = np.zeros((N, Hq, D), dtype=np.float64)
    units = sorted(((s, kh) for s in range(N) for kh in range(Hkv)), key=lambda u: -int(h["sl"][u[0]]))

    def run(u):
        s, kh = u
        rows = [(s, kh * g + i) for i in range(g)]
        out[s, kh * g:(kh + 1) * g] = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale,
                                                          rows=rows)

    with ThreadPoolExecutor(max_workers=host_threads()) as ex:
        list(ex.map(run, units))
    return out


def oracle_decode_fp8_all_rows(q, kc, vc, bt, sl, ks, vs, scale) -> np.ndarray:
    """oracle.paged_decode_fp8 over a whole batch, one task per sequence on
    host threads (each task sees its own sequence's query rows, table and
    length, and the whole pools)."""
    N, Hq, D = q.shape
    out = np.zeros((N, Hq, D), dtype=np.float64)
    order = sorted(range(N), key=lambda s: -int(sl[s]))

    def run(s):
        out[s:s + 1] = oracle.paged_decode_fp8(q[s:s + 1], kc, vc, bt[s:s + 1], sl[s:s + 1], ks, vs, scale)

    with ThreadPoolExecutor(max_workers=host_threads()) as ex:
        list(ex.map(run, order))
    return out


def oracle_decode_multi_all_rows(q, kc, vc, bt, sl, qs, scale) -> np.ndarray:
    """oracle.paged_decode_multi over a whole batch, one task per sequence on
    host threads (q_start rebased to each sequence's rows)."""
    T, Hq, D = q.shape
    out = np.zeros((T, Hq, D), dtype=np.float64)
    N = len(sl)
    order = sorted(range(N), key=lambda s: -int(sl[s]) * int(qs[s + 1] - qs[s]))

    def run(s):
        a, b = int(qs[s]), int(qs[s + 1])
        if b > a:
            out[a:b] = oracle.paged_decode_multi(q[a:b], kc, vc, bt[s:s + 1], sl[s:s + 1],
                                                 np.array([0, b - a], dtype=np.int32), scale)

    with ThreadPoolExecutor(max_workers=host_threads()) as ex:
        list(ex.map(run, order))
    return out
