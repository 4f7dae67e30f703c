"""pa_decode_noalloc: the decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a plugin inside an inference engine that
owns all device memory through its own pool, a runtime whose memory budget is
fixed at start-up, or a foreign-language caller with no CUDA allocation
binding.  For them the library keeps its split-K scratch in a fixed 32 MiB
device array of its own.  These tests call that entry point through the C ABI
and check it, within the parity tolerance, against pa_decode with a
PyTorch-allocated workspace and against the fp64 oracle, on consecutive calls
(the shared buffer keeps each call's contents for the next).  The file is
named to be collected last.
"""
import numpy as np
import pytest
import torch

from helpers import assert_close, oracle_decode, to_f64
from paged_kv_cache_432_b200 import build as pa_build
from paged_kv_cache_432_b200 import pagedattn as pa
from paged_kv_cache_432_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _pair(w, pb, max_seq_len=None):
    """(noalloc output, allocating-entry output) for workload w; the no-alloc
    output buffer starts as NaN so that a row it fails to write shows."""
    msl = w.max_seq_len if max_seq_len is None else max_seq_len
    ref = pa.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                    max_seq_len=msl, partition_blocks=pb)
    out = torch.full_like(w.q, float("nan"))
    pa.decode_noalloc(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, out,
                      max_seq_len=msl, partition_blocks=pb)
    torch.cuda.synchronize()
    return out, ref


def _check(w, pb, what, max_seq_len=None):
    assert pa.workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_seq_len if max_seq_len is None else max_seq_len, pb) > 0, \
        "the case must use the scratch buffer"
    out, ref = _pair(w, pb, max_seq_len)
    assert torch.isfinite(out.float()).all(), f"{what}: a row was not written"
    assert_close(to_f64(out), to_f64(ref), w.dtype, f"{what}: noalloc vs pa_decode")
    assert_close(to_f64(out), oracle_decode(w), w.dtype, f"{what}: noalloc vs the oracle")


def test_noalloc_matches_allocating_entry_and_oracle_on_consecutive_calls():
    pa_build.build()
    pa.device_error(clear=True)
    # call 1: long sequences, split into many partitions (uses the buffer)
    w1 = wl.build([3000, 17, 1, 700, 2049], 32, 8, 128, torch.bfloat16, seed=101, device="cuda")
    _check(w1, 4, "call 1")
    # call 2: different sizes and dtype; reads partials written over call 1's
    w2 = wl.build([513, 40, 0, 1200], 8, 2, 64, torch.float32, seed=102, device="cuda")
    _check(w2, 2, "call 2")
    # call 3: call 1's shapes and bound, shorter sequences: fewer pieces per
    # unit, so call 1's later partials are still in the buffer past the ones
    # this call writes and must not be read
    w3 = wl.build([1500, 17, 1, 300, 1000], 32, 8, 128, torch.bfloat16, seed=103, device="cuda",
                  table_width=w1.max_blocks_per_seq)
    _check(w3, 4, "call 3", max_seq_len=w1.max_seq_len)
    assert pa.device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_buffer():
    pa_build.build()
    # 64 sequences x 32 heads, 2048 tokens in 1-block partitions: ~130 MiB of partials
    N, Hq, Hkv, D, L = 64, 32, 32, 128, 2048
    assert pa.workspace_size(N, Hq, Hkv, D, L, 1) > pa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((N, Hq, D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, Hkv, 16, D), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((N, L // 16), dtype=torch.int32, device="cuda")
    sl = torch.full((N,), 16, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.decode_noalloc(q, kc, kc, bt, sl, 0.1, out, max_seq_len=L, partition_blocks=1)
    assert e.value.status == pa.PA_ERR_SCRATCH_LIMIT
    assert (out == 0).all()  # nothing was launched
