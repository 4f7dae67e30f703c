"""The test helpers that run the oracle on host threads give exactly what one
plain call of the oracle gives (they only split the batch into tasks), and the
benchmark's partition setting matches the library's."""
import numpy as np
import torch

import oracle
from helpers import (host, oracle_decode, oracle_decode_all_rows, oracle_decode_fp8_all_rows,
                     oracle_decode_multi_all_rows)
from paged_kv_cache_432_b200 import workload as wl


def test_threaded_decode_equals_one_call():
    w = wl.build([35, 1, 0, 17, 300, 64], 8, 2, 64, torch.bfloat16, seed=3)
    h = host(w)
    assert np.array_equal(oracle_decode_all_rows(w, h), oracle_decode(w, h))


def test_threaded_fp8_decode_equals_one_call():
    w = wl.build([35, 1, 0, 17, 300], 8, 4, 64, torch.bfloat16, seed=4)
    kc, vc, ks, vs = (wl.as_numpy(t) for t in wl.fp8_pools(w))
    args = (wl.as_numpy(w.q), kc, vc, wl.as_numpy(w.block_tables), wl.as_numpy(w.seq_lens), ks, vs, w.scale)
    assert np.array_equal(oracle_decode_fp8_all_rows(*args), oracle.paged_decode_fp8(*args))


def test_threaded_multi_equals_one_call():
    w = wl.build([35, 20, 17, 300], 8, 2, 64, torch.bfloat16, seed=5)
    h = host(w)
    n = [3, 0, 17, 5]
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = wl.as_numpy(torch.randn((int(qs[-1]), 8, 64), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16))
    one = oracle.paged_decode_multi(q, h["kc"], h["vc"], h["bt"], h["sl"], qs, w.scale)
    assert np.array_equal(oracle_decode_multi_all_rows(q, h["kc"], h["vc"], h["bt"], h["sl"], qs, w.scale), one)


def test_bench_partition_setting_matches_the_library():
    import bench
    from paged_kv_cache_432_b200 import build as pa_build
    from paged_kv_cache_432_b200 import pagedattn as pa

    pa_build.build()
    for pb in (0, -1, 1, 32, 100):
        assert bench.resolve_partition_blocks(pb) == pa.partition_blocks(8, 8, 131072, pb)
