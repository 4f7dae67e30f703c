"""Several query tokens per sequence (speculative-decoding check, short
prefill chunks) through pa_decode_multi, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, host, to_f64
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
