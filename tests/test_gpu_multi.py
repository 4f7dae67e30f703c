"""Several query tokens per sequence (speculative-decoding check, short
prefill chunks) through pa_decode_multi, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, host, oracle_decode_multi_all_rows, to_f64
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


def _queries(n_per_seq, Hq, D, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn((sum(n_per_seq), Hq, D), generator=g, device=DEV).to(torch.bfloat16)
    qs = torch.tensor(np.concatenate([[0], np.cumsum(n_per_seq)]), dtype=torch.int32, device=DEV)
    return q, qs


def _oracle(w, q, qs):
    h = host(w)
    return oracle.paged_decode_multi(wl.as_numpy(q), h["kc"], h["vc"], h["bt"], h["sl"], qs.cpu().numpy(), w.scale)


@pytest.mark.parametrize("Hq,Hkv,nq", [(8, 2, [4, 1, 3, 2]), (4, 4, [16, 5, 9, 1]), (32, 4, [2, 1, 2, 2]),
                                       (16, 8, [8, 3, 8, 1])])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("pb", [0, 2, -1])
def test_multi_query_matches_oracle(Hq, Hkv, nq, D, pb):
    lens = [35, 17, 700, 1500]
    w = wl.build(lens, Hq, Hkv, D, torch.bfloat16, seed=Hq + D, device=DEV, poison_unused=True)
    q, qs = _queries(nq, Hq, D, seed=len(nq) + D)
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max(nq),
                          max_seq_len=w.max_seq_len, partition_blocks=pb)
    torch.cuda.synchronize()
    assert_close(to_f64(out), _oracle(w, q, qs), torch.bfloat16, f"multi {Hq}/{Hkv} D={D} pb={pb}")
    assert pa.device_error() == 0


def test_one_query_token_each_is_bitwise_the_decode():
    w = wl.build([35, 1, 16, 17, 900], 32, 8, 128, torch.bfloat16, seed=3, device=DEV)
    qs = torch.arange(w.num_seqs + 1, dtype=torch.int32, device=DEV)
    a = pa.decode_multi(w.q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, 1,
                        max_seq_len=w.max_seq_len)
    b = pa.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_too_many_query_tokens_are_flagged():
    w = wl.build([40, 40], 8, 2, 128, torch.bfloat16, seed=4, device=DEV)
    q, qs = _queries([2, 5], 8, 128, seed=4)  # the second sequence has 5 > max_q_len = 4
    pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, 4, max_seq_len=40)
    assert pa.device_error() & pa.PA_DEVERR_SEQ_LEN


# ------------------------------------------------------------------ prefill chunks (tile kernel)
PREFILL_CASES = [
    # lens, new tokens per sequence: chunks of 64..512, chunks that start
    # mid-block, a whole sequence (n = L), an empty sequence
    ([700, 513, 64, 1000, 300, 0], [64, 100, 64, 512, 300, 0]),
    ([4100, 77, 2049], [257, 77, 129]),
]


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (64, 8), (6, 1), (16, 16)])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("case", [0, 1])
def test_prefill_chunks_match_oracle(Hq, Hkv, D, case):
    """More (query token, head) rows per sequence than one MMA fragment: the
    tensor-memory tile kernel, causal among the new tokens; unused slots hold
    NaN (a slot past a sequence's length must not reach the output)."""
    lens, nq = PREFILL_CASES[case]
    w = wl.build(lens, Hq, Hkv, D, torch.bfloat16, seed=Hq + D + case, device=DEV, poison_unused=True)
    q, qs = _queries(nq, Hq, D, seed=Hq + case)
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max(nq),
                          max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert_close(to_f64(out), _oracle(w, q, qs), torch.bfloat16, f"prefill {Hq}/{Hkv} D={D} case {case}")


def test_prefill_many_sequences_without_key_chunks():
    """Enough tiles to fill the device without cutting the keys: every row is
    written by its tile directly (no merge)."""
    rng = np.random.default_rng(4)
    lens = [int(x) for x in rng.integers(300, 2500, size=24)]
    nq = [min(L, int(x)) for L, x in zip(lens, rng.integers(64, 400, size=24))]
    w = wl.build(lens, 32, 8, 128, torch.bfloat16, seed=77, device=DEV, poison_unused=True)
    q, qs = _queries(nq, 32, 128, seed=5)
    assert pa.multi_workspace_size(w.num_seqs, q.shape[0], 32, 8, 128, w.max_seq_len) >= 0
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max(nq),
                          max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    h = host(w)
    ref = oracle_decode_multi_all_rows(wl.as_numpy(q), h["kc"], h["vc"], h["bt"], h["sl"], qs.cpu().numpy(), w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "prefill, 24 sequences")


def test_prefill_long_sequences_cut_into_balancing_chunks():
    """Long sequences with enough tiles to fill the device: the keys are still
    cut, into chunks of at least 256 blocks, so that more, shorter items even
    out the SMs' work; each row merges its chunks."""
    from test_abi import _tile_splits

    rng = np.random.default_rng(9)
    lens = [int(x) for x in rng.integers(8300, 9000, size=10)]
    nq = [128] * 10
    w = wl.build(lens, 16, 2, 128, torch.bfloat16, seed=79, device=DEV, poison_unused=True)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    work_tiles = (-(-sum(nq) // 32) + len(lens)) * 2  # tiles of 2 x 16 tokens x 8 heads, per kv head
    assert _tile_splits(sms, work_tiles, -(-w.max_seq_len // 16)) >= 2
    q, qs = _queries(nq, 16, 128, seed=9)
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max(nq),
                          max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    h = host(w)
    ref = oracle_decode_multi_all_rows(wl.as_numpy(q), h["kc"], h["vc"], h["bt"], h["sl"], qs.cpu().numpy(), w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "prefill, long sequences in balancing chunks")


def test_prefill_more_tokens_than_max_q_len_are_flagged():
    w = wl.build([300, 300], 32, 8, 128, torch.bfloat16, seed=6, device=DEV)
    q, qs = _queries([64, 100], 32, 128, seed=6)  # 100 > max_q_len = 80
    out = torch.full_like(q, float("nan"))
    pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, 80, out=out,
                    max_seq_len=300)
    torch.cuda.synchronize()
    assert pa.device_error() & pa.PA_DEVERR_SEQ_LEN
    # the rows within the bound are exact: sequence 0 whole, and sequence 1's
    # first 80 query rows as its last 80 positions; its excess rows are not written
    assert torch.isnan(out[144:164].float()).all()
    h = host(w)
    ref0 = oracle.paged_decode_multi(wl.as_numpy(q)[:64], h["kc"], h["vc"], h["bt"][:1], h["sl"][:1],
                                     np.array([0, 64], np.int32), w.scale)
    assert_close(to_f64(out)[:64], ref0, torch.bfloat16, "prefill seq 0")
    ref1 = oracle.paged_decode_multi(wl.as_numpy(q)[64:144], h["kc"], h["vc"], h["bt"][1:2],
                                     np.array([300], np.int32), np.array([0, 80], np.int32), w.scale)
    assert_close(to_f64(out)[64:144], ref1, torch.bfloat16, "prefill seq 1, clamped")


def test_prefill_more_sequences_than_one_launch_holds():
    """More sequences than one tile-kernel launch takes (256): several launches
    over consecutive ranges of sequences, each with its own work counter."""
    rng = np.random.default_rng(9)
    lens = [int(x) for x in rng.integers(20, 300, size=300)]
    nq = [min(L, int(x)) for L, x in zip(lens, rng.integers(5, 40, size=300))]
    w = wl.build(lens, 16, 4, 64, torch.bfloat16, seed=12, device=DEV, poison_unused=True)
    q, qs = _queries(nq, 16, 64, seed=12)
    out = pa.decode_multi(q, qs, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, max(nq),
                          max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    h = host(w)
    ref = oracle_decode_multi_all_rows(wl.as_numpy(q), h["kc"], h["vc"], h["bt"], h["sl"], qs.cpu().numpy(), w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "prefill, 300 sequences")
