"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the same
seeded inputs.  Cache writes and block-table indexing are compared bit for bit;
attention outputs within max-abs 2e-2 / normwise max-rel 1e-2 (bf16) or
max-abs 1e-5 (fp32)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, gpu_decode, host, oracle_decode, oracle_decode_all_rows, to_f64
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


def _bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


# ------------------------------------------------------------------ cache write
@pytest.mark.parametrize("name", ["tiny", "mha", "gqa"])
def test_cache_write_bit_exact(name):
    w = wl.make(name, device=DEV)
    h = host(w)
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    pa.cache_write(w.new_k, w.new_v, w.slot_mapping, kc, vc)
    torch.cuda.synchronize()
    kc_o, vc_o, bad = oracle.cache_write(h["nk"], h["nv"], h["sm"], h["kc"], h["vc"])
    assert bad == 0
    assert np.array_equal(_bits(wl.as_numpy(kc)), _bits(kc_o))
    assert np.array_equal(_bits(wl.as_numpy(vc)), _bits(vc_o))
    assert pa.device_error() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128])
def test_cache_write_padding_sentinel_and_out_of_range(dtype, D):
    g = torch.Generator(device=DEV).manual_seed(5)
    NB, H, T = 6, 3, 40
    sentinel = torch.full((NB, H, 16, D), 7.0, dtype=dtype, device=DEV)
    k = torch.randn((T, H, D), generator=g, device=DEV).to(dtype)
    v = torch.randn((T, H, D), generator=g, device=DEV).to(dtype)
    slots = torch.randperm(NB * 16, generator=torch.Generator().manual_seed(1))[:T].to(torch.int64)
    slots[::7] = -1
    slots[5] = NB * 16 + 3  # outside the pool: skipped and flagged
    slots = slots.to(DEV)
    kc, vc = sentinel.clone(), sentinel.clone()
    pa.cache_write(k, v, slots, kc, vc)
    torch.cuda.synchronize()
    kc_o, vc_o, bad = oracle.cache_write(wl.as_numpy(k), wl.as_numpy(v), wl.as_numpy(slots),
                                         wl.as_numpy(sentinel), wl.as_numpy(sentinel))
    assert bad == 1
    assert np.array_equal(_bits(wl.as_numpy(kc)), _bits(kc_o))
    assert np.array_equal(_bits(wl.as_numpy(vc)), _bits(vc_o))
    assert pa.device_error() == pa.PA_DEVERR_SLOT_OOB


# ------------------------------------------------------------------ decode, full compare
@pytest.mark.parametrize("pb", [0, -1, 1, 2])
def test_tiny_fp32(pb):
    """The tiny check (lens {35,1,16,17}, fp32, D=64, 2 q heads on 1 kv head)
    after the cache write of each sequence's newest token."""
    w = wl.make("tiny", device=DEV)
    h = host(w)
    pa.cache_write(w.new_k, w.new_v, w.slot_mapping, w.k_cache, w.v_cache)
    h["kc"], h["vc"], _ = oracle.cache_write(h["nk"], h["nv"], h["sm"], h["kc"], h["vc"])
    out = gpu_decode(w, partition_blocks=pb)
    ref = oracle_decode(w, h)
    assert_close(to_f64(out), ref, torch.float32, f"tiny pb={pb}")
    assert pa.device_error() == 0


EDGE_LENS = [1, 15, 16, 17, 0, 511, 512, 513, 33, 1000]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 2), (8, 2), (32, 8), (16, 2), (32, 2)])
@pytest.mark.parametrize("pb", [0, -1, 3, 32])
def test_edge_lengths(dtype, D, Hq, Hkv, pb):
    """Lengths at block and partition edges (and an empty sequence), group sizes
    1..16, both head sizes, split and unsplit."""
    w = wl.build(EDGE_LENS, Hq, Hkv, D, dtype, seed=D + Hq + Hkv, device=DEV, poison_unused=True)
    out = gpu_decode(w, partition_blocks=pb)
    ref = oracle_decode(w)
    assert_close(to_f64(out), ref, dtype, f"edge {dtype} D={D} {Hq}/{Hkv} pb={pb}")
    assert (to_f64(out)[EDGE_LENS.index(0)] == 0).all()
    assert pa.device_error() == 0


@pytest.mark.parametrize("name,Hq,Hkv", [("mha", 32, 32), ("gqa", 32, 8), ("long", 64, 8)])
def test_config_shapes_reduced_lengths(name, Hq, Hkv):
    """Each config's head layout on lengths the oracle covers in full (several
    tiles per sequence and ragged tails), in the config's partition setting."""
    rng = np.random.default_rng(3)
    lens = [int(x) for x in rng.integers(1, 3000, size=12)] + [2048, 4097]
    w = wl.build(lens, Hq, Hkv, 128, torch.bfloat16, seed=11, device=DEV,
                 partition_blocks=32 if name == "long" else 0)
    out = gpu_decode(w)
    assert_close(to_f64(out), oracle_decode(w), torch.bfloat16, name)


# ------------------------------------------------------------------ invariances (bitwise on the GPU)
def test_physical_permutation_is_bitwise_invariant():
    w = wl.build([35, 1, 16, 17, 700, 1500, 96], 32, 8, 128, torch.bfloat16, seed=21, device=DEV)
    base = gpu_decode(w)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(2)).to(DEV)
    kc = torch.empty_like(w.k_cache)
    vc = torch.empty_like(w.v_cache)
    kc[perm] = w.k_cache
    vc[perm] = w.v_cache
    bt = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(), w.block_tables)
    moved = gpu_decode(w, k_cache=kc, v_cache=vc, block_tables=bt)
    assert torch.equal(base.view(torch.int16), moved.view(torch.int16))


@pytest.mark.parametrize("prefix_len", [4096, 4090])
def test_shared_prefix_matches_private_copies_bitwise(prefix_len):
    """Sequences sharing prefix blocks give the same bits as the same sequences
    holding private copies of every block (and, within tolerance, the oracle)."""
    w = wl.make("prefix", device=DEV, prefix_len=prefix_len)
    shared = gpu_decode(w)
    refs = [b for t in w.tables_host for b in t]
    src = torch.tensor(refs, dtype=torch.long, device=DEV)
    kc = w.k_cache[src].contiguous()
    vc = w.v_cache[src].contiguous()
    bt = torch.full_like(w.block_tables, -1)
    i = 0
    for s, t in enumerate(w.tables_host):
        bt[s, : len(t)] = torch.arange(i, i + len(t), dtype=torch.int32, device=DEV)
        i += len(t)
    private = gpu_decode(w, k_cache=kc, v_cache=vc, block_tables=bt)
    assert torch.equal(shared.view(torch.int16), private.view(torch.int16))
    assert_close(to_f64(shared), oracle_decode_all_rows(w), torch.bfloat16, "prefix, every row")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_nan_in_unreachable_slots_changes_nothing(dtype):
    lens = [35, 1, 16, 17, 513, 250]
    clean = wl.build(lens, 8, 2, 128, dtype, seed=31, device=DEV)
    dirty = wl.build(lens, 8, 2, 128, dtype, seed=31, device=DEV, poison_unused=True)
    assert torch.isnan(dirty.k_cache.float()).any()
    a, b = gpu_decode(clean, partition_blocks=4), gpu_decode(dirty, partition_blocks=4)
    assert torch.isfinite(b.float()).all()
    assert torch.equal(a, b)


@pytest.mark.parametrize("pb", [1, 4, 32])
def test_split_and_single_pass_agree(pb):
    w = wl.build([3000, 600, 17, 4096], 64, 8, 128, torch.bfloat16, seed=41, device=DEV)
    ref = oracle_decode(w)
    single = gpu_decode(w, partition_blocks=-1)
    split = gpu_decode(w, partition_blocks=pb)
    assert_close(to_f64(single), ref, torch.bfloat16, "single")
    assert_close(to_f64(split), ref, torch.bfloat16, f"split pb={pb}")


@pytest.mark.parametrize("lens,Hq,Hkv", [([30000, 5, 700, 0, 64], 8, 1), ([70000], 16, 2),
                                          ([1] * 300 + [9000], 4, 4)])
def test_balanced_split_long_unit_across_many_warps(lens, Hq, Hkv):
    """Balanced split (partition_blocks = 0): a long unit is cut at warp-range
    boundaries into many pieces, next to units that are one piece."""
    w = wl.build(lens, Hq, Hkv, 128, torch.bfloat16, seed=sum(lens) % 1000, device=DEV)
    out = gpu_decode(w, partition_blocks=0)
    assert_close(to_f64(out), oracle_decode(w), torch.bfloat16, f"balanced {lens[:3]}")
    assert pa.device_error() == 0


# ------------------------------------------------------------------ shared-prefix decode
def _shared_prefix_decode(w, pb=0, **kw):
    out = pa.decode_shared_prefix(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                  w.shared_prefix_blocks, max_seq_len=w.max_seq_len, partition_blocks=pb, **kw)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("prefix_len,suffixes,Hq,Hkv,D", [
    (64, [5, 40, 17, 0, 200], 8, 2, 128),
    (4096, [64, 1, 300, 512, 16], 32, 8, 128),
    (4090, [5, 40, 700], 16, 2, 64),        # prefix ends mid-block: 255 shared blocks + private copies
    (1600, [33] * 40, 4, 4, 128),           # many sequences: several row tiles per kv head
    (512, [9, 100], 32, 2, 128),            # group of 16
])
@pytest.mark.parametrize("pb", [0, 4])
def test_shared_prefix_decode_matches_oracle(prefix_len, suffixes, Hq, Hkv, D, pb):
    lens = [prefix_len + x for x in suffixes]
    w = wl.build(lens, Hq, Hkv, D, torch.bfloat16, seed=prefix_len + len(lens), device=DEV,
                 prefix_len=prefix_len, poison_unused=True)
    assert w.shared_prefix_blocks == prefix_len // 16
    out = _shared_prefix_decode(w, pb)
    assert_close(to_f64(out), oracle_decode(w), torch.bfloat16, f"shared prefix {prefix_len}")
    assert pa.device_error() == 0


def test_shared_prefix_preconditions_are_flagged():
    w = wl.build([600, 700], 8, 2, 128, torch.bfloat16, seed=5, device=DEV, prefix_len=512)
    bt = w.block_tables.clone()
    bt[1, 3] = w.tables_host[1][-1]  # sequence 1 no longer starts with the shared blocks
    pa.decode_shared_prefix(w.q, w.k_cache, w.v_cache, bt, w.seq_lens, w.scale, 32, max_seq_len=700)
    assert pa.device_error() & pa.PA_DEVERR_PREFIX
    short = w.seq_lens.clone()
    short[0] = 100  # shorter than the prefix
    pa.decode_shared_prefix(w.q, w.k_cache, w.v_cache, w.block_tables, short, w.scale, 32, max_seq_len=700)
    assert pa.device_error() & pa.PA_DEVERR_PREFIX


def test_shared_prefix_block_outside_the_pool_is_masked_and_flagged():
    """A shared block id outside the pool (in every table, so the prefix stays
    shared): flagged, its tokens take no part, the rest is exact attention."""
    lens = [160 + x for x in (40, 3, 97)]
    w = wl.build(lens, 8, 2, 128, torch.bfloat16, seed=91, device=DEV, prefix_len=160, poison_unused=True)
    bt = w.block_tables.clone()
    bt[:, 3] = w.num_blocks + 7
    out = pa.decode_shared_prefix(w.q, w.k_cache, w.v_cache, bt, w.seq_lens, w.scale, w.shared_prefix_blocks,
                                  max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() & pa.PA_DEVERR_BLOCK_OOB
    assert torch.isfinite(out.float()).all()
    h = host(w)
    for s, L in enumerate(lens):
        keep = [t for t in range(L) if t // 16 != 3]
        nb = -(-len(keep) // 16)
        packed_k = np.zeros((nb, 2, 16, 128), np.uint16)
        packed_v = np.zeros_like(packed_k)
        for i, t in enumerate(keep):
            b = w.tables_host[s][t // 16]
            packed_k[i // 16, :, i % 16] = h["kc"][b, :, t % 16]
            packed_v[i // 16, :, i % 16] = h["vc"][b, :, t % 16]
        ref = oracle.paged_decode(h["q"][s:s + 1], packed_k, packed_v, np.arange(nb, dtype=np.int32)[None, :],
                                  np.array([len(keep)], np.int32), w.scale)
        assert_close(to_f64(out)[s:s + 1], ref, torch.bfloat16, f"seq {s} without the bad shared block")


# ------------------------------------------------------------------ the two steps separately
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_partition_partials_match_oracle(dtype):
    """pa_decode_partitions alone: the workspace partials (m, l, acc) of every
    partition against the oracle's split-K form."""
    pb = 4
    w = wl.build([300, 64, 65, 17], 8, 2, 128, dtype, seed=51, device=DEV)
    msl = w.max_seq_len
    ws = pa.alloc_workspace(w.num_seqs, 8, 2, 128, msl, pb, device=DEV)
    ws.fill_(0)
    out = torch.zeros_like(w.q)
    pa.decode_partitions(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, out, msl, pb, ws)
    torch.cuda.synchronize()
    h = host(w)
    m_o, l_o, acc_o, np_o = oracle.decode_partials(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, pb * 16)
    P = -(-(-(-msl // 16)) // pb)  # ceil(ceil(msl / 16) / pb)
    m_g, l_g, acc_g = (t.double().cpu().numpy() for t in pa.workspace_views(ws, w.num_seqs, 8, 128, P)[:3])
    for s, L in enumerate(w.lens_host):
        n = int(np_o[s])
        if n <= 1:  # written straight to out
            assert_close(to_f64(out)[s], (acc_o[s, :, 0] / l_o[s, :, 0, None]), dtype, "single-part row")
            continue
        tol = 2e-2 if dtype == torch.bfloat16 else 1e-5
        np.testing.assert_allclose(m_g[s, :, :n], m_o[s, :, :n], rtol=0, atol=tol)
        # normalised partition outputs and weights
        assert_close(acc_g[s, :, :n] / l_g[s, :, :n, None], acc_o[s, :, :n] / l_o[s, :, :n, None], dtype, "acc/l")
        lw_g = l_g[s, :, :n] * np.exp(m_g[s, :, :n] - m_o[s, :, :n])
        np.testing.assert_allclose(lw_g, l_o[s, :, :n], rtol=1e-2 if dtype == torch.bfloat16 else 1e-5)


def test_reduce_of_oracle_partials_matches_oracle_merge():
    """pa_decode_reduce alone, fed with the oracle's own partials (fp32)."""
    pb = 2
    w = wl.build([100, 500, 33, 64, 7], 16, 4, 64, torch.float32, seed=61, device=DEV)
    msl = w.max_seq_len
    h = host(w)
    m_o, l_o, acc_o, np_o = oracle.decode_partials(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, pb * 16)
    P = -(-(-(-msl // 16)) // pb)  # ceil(ceil(msl / 16) / pb)
    ws = pa.alloc_workspace(w.num_seqs, 16, 4, 64, msl, pb, device=DEV)
    m_v, l_v, acc_v, parts_v = pa.workspace_views(ws, w.num_seqs, 16, 64, P, num_kv_heads=4)
    m_v.zero_(), l_v.zero_(), acc_v.zero_()
    parts_v[:] = torch.from_numpy(np_o).int().to(DEV)[:, None]  # pieces of every kv head
    Po = m_o.shape[2]
    m_v[:, :, :Po] = torch.from_numpy(m_o).float().to(DEV)
    l_v[:, :, :Po] = torch.from_numpy(l_o).float().to(DEV)
    acc_v[:, :, :Po] = torch.from_numpy(acc_o).float().to(DEV)
    out = torch.full_like(w.q, 123.0)
    pa.decode_reduce(w.seq_lens, out, 4, w.max_blocks_per_seq, msl, pb, ws)
    torch.cuda.synchronize()
    ref = oracle.lse_merge(m_o, l_o, acc_o, np_o)
    g = to_f64(out)
    for s in range(w.num_seqs):
        if np_o[s] <= 1:
            assert (g[s] == 123.0).all()  # left to the partition step
        else:
            np.testing.assert_allclose(g[s], ref[s], rtol=0, atol=2e-6)


# ------------------------------------------------------------------ limits and device-side errors
def test_many_sequences_span_several_launches():
    """More sequences than one launch's item table holds (2048)."""
    rng = np.random.default_rng(71)
    lens = [int(x) for x in rng.integers(0, 80, size=2500)]
    w = wl.build(lens, 4, 1, 64, torch.bfloat16, seed=71, device=DEV)
    out = gpu_decode(w, partition_blocks=2)
    assert_close(to_f64(out), oracle_decode(w), torch.bfloat16, "2500 seqs")


def test_out_of_pool_block_id_is_masked_and_flagged():
    w = wl.build([40, 40], 4, 1, 128, torch.bfloat16, seed=81, device=DEV)
    bt = w.block_tables.clone()
    bt[1, 1] = w.num_blocks + 5  # second block of sequence 1 points outside the pool
    out = gpu_decode(w, block_tables=bt)
    assert pa.device_error() & pa.PA_DEVERR_BLOCK_OOB
    assert torch.isfinite(out.float()).all()
    # sequence 0 is untouched by the bad entry
    ref = oracle_decode(w, rows=[(0, i) for i in range(4)])
    assert_close(to_f64(out)[0], ref, torch.bfloat16, "seq 0")
    # sequence 1 equals attention over its remaining tokens (blocks 0 and 2),
    # packed into a fresh two-block pool for the oracle
    h = host(w)
    keep = [t for t in range(40) if t // 16 != 1]
    packed_k = np.zeros((2, 1, 16, 128), np.uint16)
    packed_v = np.zeros_like(packed_k)
    for i, t in enumerate(keep):
        b = w.tables_host[1][t // 16]
        packed_k[i // 16, 0, i % 16] = h["kc"][b, 0, t % 16]
        packed_v[i // 16, 0, i % 16] = h["vc"][b, 0, t % 16]
    ref1 = oracle.paged_decode(h["q"][1:2], packed_k, packed_v, np.array([[0, 1]], np.int32),
                               np.array([len(keep)], np.int32), w.scale)
    assert_close(to_f64(out)[1:2], ref1, torch.bfloat16, "seq 1 without the bad block")


def test_sequence_longer_than_bound_is_clamped_and_flagged():
    w = wl.build([100, 600], 4, 2, 128, torch.bfloat16, seed=91, device=DEV)
    out = gpu_decode(w, max_seq_len=300, partition_blocks=4)
    assert pa.device_error() & pa.PA_DEVERR_SEQ_LEN
    h = host(w)
    h["sl"] = np.array([100, 300], np.int32)
    ref = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "clamped")


# ------------------------------------------------------------------ several prompt groups
GROUP_CASES = [
    # (count, prefix tokens) per group, suffix lengths
    ([(3, 4096), (2, 0), (5, 1600), (1, 64)], [64, 1, 300, 512, 16, 5, 40, 700, 33, 0, 90]),
    ([(20, 512), (20, 4090)], [int(x) for x in np.random.default_rng(1).integers(1, 400, 40)]),
]


@pytest.mark.parametrize("case", [0, 1])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (16, 2, 64), (8, 8, 128)])
@pytest.mark.parametrize("pb", [0, 4])
def test_shared_prefix_groups_match_oracle(case, Hq, Hkv, D, pb):
    """Several prompt groups in one batch (a group that shares nothing, a
    prompt ending mid-block with copy-on-write, a one-sequence group), each
    group's shared blocks read once per tile of its query rows."""
    groups, suffixes = GROUP_CASES[case]
    lens, i = [], 0
    for count, pl in groups:
        lens += [pl + suffixes[i + k] for k in range(count)]
        i += count
    w = wl.build(lens, Hq, Hkv, D, torch.bfloat16, seed=case + Hq, device=DEV, groups=groups, poison_unused=True)
    maxs = max(w.group_blocks_host)
    out = pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                         w.group_start, w.group_blocks, maxs, max_seq_len=w.max_seq_len,
                                         partition_blocks=pb)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode(w), torch.bfloat16, f"groups case {case} {Hq}/{Hkv} D={D} pb={pb}")


def test_shared_prefix_groups_four_prompts_full_size():
    """The prefix-sharing workload with four prompts of 4096 tokens, each shared
    by 32 sequences, after the cache write; every row against the oracle."""
    w = wl.make("prefix", device=DEV, prompt_groups=4)
    h = host(w)
    pa.cache_write(w.new_k, w.new_v, w.slot_mapping, w.k_cache, w.v_cache)
    oracle.cache_write(h["nk"], h["nv"], h["sm"], h["kc"], h["vc"], inplace=True)
    out = pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                         w.group_start, w.group_blocks, max(w.group_blocks_host),
                                         max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode_all_rows(w, h), torch.bfloat16, "four prompts, every row")


def test_shared_prefix_more_items_than_sms():
    """1280 sequences (one query head per kv head, 32 kv heads) sharing a
    64-token prompt: 5 row tiles x 32 kv heads = 160 tile items, more than
    the SMs, so the tiles claim items from the workspace counter, which the
    call zeroes before the private blocks' decode that runs first."""
    lens = [64 + 1 + (i * 37) % 120 for i in range(1280)]
    w = wl.build(lens, 32, 32, 128, torch.bfloat16, seed=71, device=DEV, prefix_len=64, poison_unused=True)
    out = _shared_prefix_decode(w)
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode_all_rows(w), torch.bfloat16, "shared prefix, 160 tile items")


def test_shared_prefix_decode_in_several_launches():
    """More sequences (2100) than one decode launch holds (2048): the private
    blocks' decode runs as two grids, then the prefix tiles (which wait for
    the last of them only at their end), then the merge."""
    lens = [32 + 1 + (i * 13) % 60 for i in range(2100)]
    w = wl.build(lens, 8, 2, 128, torch.bfloat16, seed=72, device=DEV, prefix_len=32, poison_unused=True)
    out = _shared_prefix_decode(w)
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode_all_rows(w), torch.bfloat16, "shared prefix, two decode launches")


def test_shared_prefix_groups_more_than_one_tile_launch_holds():
    """300 prompt groups, more units than one tile launch holds (256): the
    tiles run first, in two launches, then the decode and the merge."""
    groups = [(1 + i % 2, 32 + 16 * (i % 3)) for i in range(300)]
    lens = [pl + 1 + (7 * len(groups) + 3 * k + i) % 50 for i, (count, pl) in enumerate(groups) for k in range(count)]
    w = wl.build(lens, 8, 2, 128, torch.bfloat16, seed=73, device=DEV, groups=groups, poison_unused=True)
    out = pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                         w.group_start, w.group_blocks, max(w.group_blocks_host),
                                         max_seq_len=w.max_seq_len)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert_close(to_f64(out), oracle_decode_all_rows(w), torch.bfloat16, "300 prompt groups")


def test_shared_prefix_groups_bad_group_list_is_flagged():
    w = wl.build([600, 700, 300], 8, 2, 128, torch.bfloat16, seed=5, device=DEV, groups=[(2, 512), (1, 0)])
    # a count above the bound
    gb = torch.tensor([40, 0], dtype=torch.int32, device=DEV)
    pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                   w.group_start, gb, 32, max_seq_len=700)
    assert pa.device_error() & pa.PA_DEVERR_PREFIX
    # groups out of order
    gs = torch.tensor([0, 3, 2], dtype=torch.int32, device=DEV)
    pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale,
                                   gs, w.group_blocks, 32, max_seq_len=700)
    assert pa.device_error() & pa.PA_DEVERR_PREFIX
    # a table of group 0 that does not start with the group's blocks
    bt = w.block_tables.clone()
    bt[1, 2] = w.tables_host[2][0]
    pa.decode_shared_prefix_groups(w.q, w.k_cache, w.v_cache, bt, w.seq_lens, w.scale,
                                   w.group_start, w.group_blocks, 32, max_seq_len=700)
    assert pa.device_error() & pa.PA_DEVERR_PREFIX
