"""Every output row of the full-size workloads against the fp64 oracle.

Each workload runs at full size, in the launch configuration the benchmark
times: the cache write of every sequence's newest token, then the decode with
the workload's partition setting (balanced split for mha / gqa / prefix,
32-block partitions and the log-sum-exp merge for long), through the C ABI.
The updated pools are compared bit for bit with the oracle's scatter, and
every (sequence, query head) row of the output with the oracle's attention
(bf16 bound: max-abs 2e-2 and normwise max-rel 1e-2).  The oracle runs one
task per (sequence, kv head), or per sequence, on host threads; it is the
same plain oracle as everywhere else.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import (assert_close, host, oracle_decode_all_rows, oracle_decode_fp8_all_rows,
                     oracle_decode_multi_all_rows, to_f64)
from paged_kv_cache_432_b200 import build as pa_build
from paged_kv_cache_432_b200 import pagedattn as pa
from paged_kv_cache_432_b200 import workload as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean():
    if torch.cuda.is_available():
        pa_build.build()
        pa.device_error(clear=True)
    yield
    if torch.cuda.is_available():
        torch.cuda.empty_cache()


def _bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def _write_and_check(w, h):
    """GPU cache write of the newest tokens, the same scatter by the oracle on
    the host copy (in place); the two pools must agree bit for bit."""
    pa.cache_write(w.new_k, w.new_v, w.slot_mapping, w.k_cache, w.v_cache)
    _, _, bad = oracle.cache_write(h["nk"], h["nv"], h["sm"], h["kc"], h["vc"], inplace=True)
    assert bad == 0
    assert np.array_equal(_bits(wl.as_numpy(w.k_cache)), _bits(h["kc"])), "K pool after the write"
    assert np.array_equal(_bits(wl.as_numpy(w.v_cache)), _bits(h["vc"])), "V pool after the write"


@pytest.mark.parametrize("name", ["mha", "gqa", "long"])
def test_every_row_of_the_full_size_workload(name):
    w = wl.make(name, device=DEV)
    h = host(w)
    _write_and_check(w, h)
    out = pa.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                    max_seq_len=w.max_seq_len, partition_blocks=w.partition_blocks)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode_all_rows(w, h), torch.bfloat16, f"{name}, every row")


def test_every_row_of_the_prefix_workload_both_paths():
    """The prefix-sharing workload: the shared-prefix decode (the benchmark's
    path) and the plain decode, every row of each against the oracle."""
    w = wl.make("prefix", device=DEV)
    h = host(w)
    _write_and_check(w, h)
    shared = pa.decode_shared_prefix(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                     w.shared_prefix_blocks, max_seq_len=w.max_seq_len)
    plain = pa.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    ref = oracle_decode_all_rows(w, h)
    assert_close(to_f64(shared), ref, torch.bfloat16, "prefix, shared-prefix decode, every row")
    assert_close(to_f64(plain), ref, torch.bfloat16, "prefix, plain decode, every row")


@pytest.mark.parametrize("name", ["mha", "gqa", "prefix", "long"])
def test_every_row_of_the_full_size_workload_e4m3(name):
    """The same over E4M3 pools: the quantising write of the newest tokens
    (every code of the pool compared with the oracle's quantiser), then the
    E4M3 decode in the workload's partition setting."""
    w = wl.make(name, device=DEV)
    kc, vc, ks, vs = wl.fp8_pools(w)
    w.k_cache = w.v_cache = None
    torch.cuda.empty_cache()
    kc_h, vc_h = wl.as_numpy(kc), wl.as_numpy(vc)
    kis, vis = (1.0 / ks).float(), (1.0 / vs).float()
    pa.cache_write_fp8(w.new_k, w.new_v, w.slot_mapping, kc, vc, kis, vis)
    out = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len,
                        partition_blocks=w.partition_blocks)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    kc_o, vc_o, bad = oracle.cache_write_fp8(wl.as_numpy(w.new_k), wl.as_numpy(w.new_v), wl.as_numpy(w.slot_mapping),
                                             kc_h, vc_h, wl.as_numpy(kis), wl.as_numpy(vis))
    assert bad == 0
    del kc_h, vc_h
    assert np.array_equal(wl.as_numpy(kc), kc_o) and np.array_equal(wl.as_numpy(vc), vc_o), "E4M3 pools"
    ref = oracle_decode_fp8_all_rows(wl.as_numpy(w.q), kc_o, vc_o, wl.as_numpy(w.block_tables),
                                     wl.as_numpy(w.seq_lens), wl.as_numpy(ks), wl.as_numpy(vs), w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, f"{name} E4M3, every row")


def test_every_row_of_the_speculative_check_on_the_gqa_workload():
    """The GQA workload at full size with 4 query tokens per sequence (the
    check of 3 drafted tokens + 1), every (query token, head) row."""
    w = wl.make("gqa", device=DEV)
    g = torch.Generator(device=DEV).manual_seed(9)
    q = torch.randn((4 * w.num_seqs, w.num_q_heads, w.head_dim), generator=g, device=DEV).to(torch.bfloat16)
    qs = torch.arange(0, 4 * w.num_seqs + 1, 4, dtype=torch.int32, device=DEV)
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, 4,
                          max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    h = host(w)
    ref = oracle_decode_multi_all_rows(wl.as_numpy(q), h["kc"], h["vc"], h["bt"], h["sl"], qs.cpu().numpy(), w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "gqa, 4 query tokens, every row")
