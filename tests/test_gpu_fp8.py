"""FP8 E4M3 KV cache: the quantising cache write and decode over E4M3 pools,
through the C ABI, against the oracle's E4M3 codec and fp64 attention over the
decoded values.  Codes are compared bit for bit (every bf16 bit pattern goes
through the quantiser); attention outputs within max-abs 2e-2 / normwise
max-rel 1e-2, the bf16 bound (q and out are bf16)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, to_f64
from paged_kv_cache_432_b200 import pagedattn as pa
from paged_kv_cache_432_b200 import workload as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean_error_word():
    if torch.cuda.is_available():
        from paged_kv_cache_432_b200 import build

        build.build()
        pa.device_error(clear=True)
    yield


def _np(t):
    return wl.as_numpy(t)


# ------------------------------------------------------------------ quantising cache write
INV_SCALES = [1.0, 1.0 / 3.0, 2.0 ** -7, 5.5, 300.0, 1e-30]


@pytest.mark.parametrize("D", [64, 128])
def test_cache_write_fp8_every_bf16_pattern(D):
    """All 65536 bf16 bit patterns (zeros of both signs, subnormals, ties,
    values past 448, infinities, NaNs) times six inverse scales, one per kv
    head, quantised into a pool prefilled with a sentinel; padding slots and
    untouched slots keep the sentinel."""
    H = len(INV_SCALES)
    T = 65536 // D
    pat = torch.from_numpy(np.arange(65536, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).reshape(T, D)
    k = pat[:, None, :].expand(T, H, D).contiguous()
    v = torch.flip(pat, dims=[0])[:, None, :].expand(T, H, D).contiguous()
    NB = (T + 8 + 15) // 16 + 2
    slots = torch.randperm(NB * 16, generator=torch.Generator().manual_seed(2))[:T].to(torch.int64)
    pad = slots.clone()
    pad[::29] = -1
    kis = torch.tensor(INV_SCALES, dtype=torch.float32)
    vis = torch.flip(kis, dims=[0]).contiguous()
    sentinel = torch.full((NB, H, 16, D), 0xA5, dtype=torch.uint8)
    kc, vc = sentinel.to(DEV), sentinel.to(DEV)
    pa.cache_write_fp8(k.to(DEV), v.to(DEV), pad.to(DEV), kc, vc, kis.to(DEV), vis.to(DEV))
    torch.cuda.synchronize()
    kc_o, vc_o, bad = oracle.cache_write_fp8(_np(k), _np(v), pad.numpy(), sentinel.numpy(), sentinel.numpy(),
                                             kis.numpy(), vis.numpy())
    assert bad == 0
    got_k, got_v = _np(kc), _np(vc)
    assert np.array_equal(got_k, kc_o), f"{int((got_k != kc_o).sum())} K codes differ"
    assert np.array_equal(got_v, vc_o), f"{int((got_v != vc_o).sum())} V codes differ"
    assert pa.device_error() == 0


def test_cache_write_fp8_out_of_range_slot_is_skipped_and_flagged():
    g = torch.Generator(device=DEV).manual_seed(4)
    NB, H, D, T = 5, 2, 128, 30
    k = torch.randn((T, H, D), generator=g, device=DEV).to(torch.bfloat16)
    v = torch.randn((T, H, D), generator=g, device=DEV).to(torch.bfloat16)
    slots = torch.randperm(NB * 16, generator=torch.Generator().manual_seed(3))[:T].to(torch.int64)
    slots[7] = NB * 16 + 1
    slots[9] = -1
    kis = torch.full((H,), 40.0)
    vis = torch.full((H,), 20.0)
    sentinel = torch.full((NB, H, 16, D), 0x3C, dtype=torch.uint8)
    kc, vc = sentinel.to(DEV), sentinel.to(DEV)
    pa.cache_write_fp8(k, v, slots.to(DEV), kc, vc, kis.to(DEV), vis.to(DEV))
    torch.cuda.synchronize()
    kc_o, vc_o, bad = oracle.cache_write_fp8(_np(k), _np(v), slots.numpy(), sentinel.numpy(), sentinel.numpy(),
                                             kis.numpy(), vis.numpy())
    assert bad == 1
    assert np.array_equal(_np(kc), kc_o) and np.array_equal(_np(vc), vc_o)
    assert pa.device_error() == pa.PA_DEVERR_SLOT_OOB


# ------------------------------------------------------------------ decode over E4M3 pools
def _fp8_case(w, poison=True):
    kc, vc, ks, vs = wl.fp8_pools(w, poison_unused=poison)
    return kc, vc, ks, vs


def _oracle_fp8(w, kc, vc, ks, vs, seqs=None):
    q, bt, sl = _np(w.q), _np(w.block_tables), _np(w.seq_lens)
    if seqs is not None:
        q, bt, sl = q[seqs], bt[seqs], sl[seqs]
    return oracle.paged_decode_fp8(q, _np(kc), _np(vc), bt, sl, _np(ks), _np(vs), w.scale)


EDGE_LENS = [1, 15, 16, 17, 0, 511, 512, 513, 33, 1000]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 2), (8, 2), (32, 8), (16, 2), (32, 2)])
@pytest.mark.parametrize("pb", [0, -1, 3, 32])
def test_fp8_decode_edge_lengths(D, Hq, Hkv, pb):
    """Block and partition edges, an empty sequence, group sizes 1..16, both
    head sizes, split and unsplit; unreachable slots hold the NaN code."""
    w = wl.build(EDGE_LENS, Hq, Hkv, D, torch.bfloat16, seed=D + Hq + 7 * Hkv, device=DEV)
    kc, vc, ks, vs = _fp8_case(w)
    out = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len,
                        partition_blocks=pb)
    torch.cuda.synchronize()
    ref = _oracle_fp8(w, kc, vc, ks, vs)
    assert_close(to_f64(out), ref, torch.bfloat16, f"fp8 D={D} {Hq}/{Hkv} pb={pb}")
    assert (to_f64(out)[EDGE_LENS.index(0)] == 0).all()
    assert pa.device_error() == 0


@pytest.mark.parametrize("Hq,Hkv", [(32, 32), (32, 8), (64, 8)])
def test_fp8_decode_ragged_lengths(Hq, Hkv):
    rng = np.random.default_rng(8)
    lens = [int(x) for x in rng.integers(1, 3000, size=12)] + [2048, 4097]
    w = wl.build(lens, Hq, Hkv, 128, torch.bfloat16, seed=19, device=DEV)
    kc, vc, ks, vs = _fp8_case(w)
    out = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert_close(to_f64(out), _oracle_fp8(w, kc, vc, ks, vs), torch.bfloat16, f"fp8 ragged {Hq}/{Hkv}")
    assert pa.device_error() == 0


@pytest.mark.parametrize("Hq,Hkv,pb", [(32, 32, 0), (32, 8, 0), (8, 2, 3), (64, 8, 32)])
def test_fp8_partitions_then_reduce_equal_the_one_call(Hq, Hkv, pb):
    """pa_decode_fp8_partitions followed by pa_decode_fp8_reduce is
    pa_decode_fp8 bit for bit (the same kernels, the merge told the E4M3
    warp ranges), and both match the oracle."""
    rng = np.random.default_rng(Hq + Hkv + pb)
    lens = [int(x) for x in rng.integers(1, 3000, size=20)] + [0, 1, 4097]
    w = wl.build(lens, Hq, Hkv, 128, torch.bfloat16, seed=23 + pb, device=DEV)
    kc, vc, ks, vs = _fp8_case(w)
    one = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len,
                        partition_blocks=pb)
    ws = pa.alloc_workspace(w.num_seqs, Hq, Hkv, 128, w.max_seq_len, pb, device=DEV)
    out = torch.full_like(w.q, float("nan"))
    pa.decode_fp8_partitions(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, out, w.max_seq_len, pb, ws)
    if ws is not None:
        pa.decode_fp8_reduce(w.seq_lens, out, Hkv, w.block_tables.shape[1], w.max_seq_len, pb, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), one.view(torch.int16))
    assert_close(to_f64(out), _oracle_fp8(w, kc, vc, ks, vs), torch.bfloat16, f"fp8 two steps {Hq}/{Hkv} pb={pb}")
    assert pa.device_error() == 0


def test_fp8_decode_scales_are_per_head():
    """Doubling one kv head's K scale changes only that head's rows; the V
    scale multiplies its rows exactly when the softmax is unchanged."""
    w = wl.build([40, 300, 17], 8, 4, 128, torch.bfloat16, seed=23, device=DEV)
    kc, vc, ks, vs = _fp8_case(w)
    base = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale).clone()
    vs2 = vs.clone()
    vs2[1] *= 2.0
    out = pa.decode_fp8(w.q, kc, vc, ks, vs2, w.block_tables, w.seq_lens, w.scale)
    torch.cuda.synchronize()
    g = w.group
    others = [h for h in range(w.num_q_heads) if h // g != 1]
    assert torch.equal(out[:, others], base[:, others])
    assert torch.equal(out[:, g:2 * g].float(), (base[:, g:2 * g].float() * 2.0))
    ks2 = ks.clone()
    ks2[2] *= 2.0
    out = pa.decode_fp8(w.q, kc, vc, ks2, vs, w.block_tables, w.seq_lens, w.scale)
    torch.cuda.synchronize()
    others = [h for h in range(w.num_q_heads) if h // g != 2]
    assert torch.equal(out[:, others], base[:, others])
    assert_close(to_f64(out), _oracle_fp8(w, kc, vc, ks2, vs), torch.bfloat16, "fp8 doubled k scale")


def test_fp8_write_then_decode_round_trip():
    """A decode step as a server runs it: quantise the new token of every
    sequence into the E4M3 pools, then decode; against the oracle's quantiser
    and fp64 attention."""
    rng = np.random.default_rng(12)
    lens = [int(x) for x in rng.integers(1, 1500, size=20)]
    w = wl.build(lens, 32, 8, 128, torch.bfloat16, seed=31, device=DEV)
    kc, vc, ks, vs = _fp8_case(w, poison=False)
    kc_h, vc_h = _np(kc), _np(vc)
    kis, vis = (1.0 / ks).float(), (1.0 / vs).float()
    pa.cache_write_fp8(w.new_k, w.new_v, w.slot_mapping, kc, vc, kis, vis)
    out = pa.decode_fp8(w.q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale)
    torch.cuda.synchronize()
    kc_o, vc_o, bad = oracle.cache_write_fp8(_np(w.new_k), _np(w.new_v), _np(w.slot_mapping), kc_h, vc_h,
                                             _np(kis), _np(vis))
    assert bad == 0
    assert np.array_equal(_np(kc), kc_o) and np.array_equal(_np(vc), vc_o)
    ref = oracle.paged_decode_fp8(_np(w.q), kc_o, vc_o, _np(w.block_tables), _np(w.seq_lens), _np(ks), _np(vs),
                                  w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "fp8 write+decode")
    assert pa.device_error() == 0


def test_fp8_decode_query_range_edges():
    """The E4M3 kernel rounds q to f16: queries near both ends of the f16
    range (tiny values that become f16 subnormals, large values up to a few
    hundred times N(0, 1)) still meet the bound; a value beyond the f16 range
    sets PA_DEVERR_Q_RANGE."""
    w = wl.build([40, 300, 17, 600], 8, 2, 128, torch.bfloat16, seed=29, device=DEV)
    kc, vc, ks, vs = _fp8_case(w)
    for factor in (1e-5, 300.0):
        q = (w.q.float() * factor).to(torch.bfloat16)
        out = pa.decode_fp8(q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len)
        torch.cuda.synchronize()
        ref = oracle.paged_decode_fp8(_np(q), _np(kc), _np(vc), _np(w.block_tables), _np(w.seq_lens), _np(ks),
                                      _np(vs), w.scale)
        assert_close(to_f64(out), ref, torch.bfloat16, f"fp8 q x {factor}")
        assert pa.device_error() == 0
    q = w.q.clone()
    q[1, 3, 5] = 7.0e4  # beyond the largest f16 value
    pa.decode_fp8(q, kc, vc, ks, vs, w.block_tables, w.seq_lens, w.scale, max_seq_len=w.max_seq_len)
    assert pa.device_error() & pa.PA_DEVERR_Q_RANGE
