"""Pins for the CPU oracle: checks against what the pages and the mathematics fix,
never against the oracle itself.

Each pin is chosen so that a plausible mistake in the oracle fails it. A wrong
gather index or layout, a dropped scale, a transposed operand, a wrong kv-head
mapping, a bad bf16 decode or a broken merge all show up in at least one test.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_432_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np_host(w):
    return dict(
        q=wl.as_numpy(w.q), kc=wl.as_numpy(w.k_cache), vc=wl.as_numpy(w.v_cache),
        bt=wl.as_numpy(w.block_tables), sl=wl.as_numpy(w.seq_lens),
    )


def _decode(w, **kw):
    h = _np_host(w)
    return oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, **kw)


# ------------------------------------------------------------------ block accounting
def test_worked_example_35_tokens():
    """The pages' worked example: 35 tokens in 16-token blocks."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_35_tokens.json")))
    L, B = g["seq_len"], g["block_size"]
    assert oracle.blocks_needed(L, B) == g["blocks"]
    assert oracle.allocated_slots(L, B) == g["allocated_slots"]
    assert oracle.unused_slots(L, B) == g["unused_slots"]
    assert round(100.0 * oracle.unused_slots(L, B) / oracle.allocated_slots(L, B)) == g["unused_percent_rounded"]


def test_only_last_block_is_partial():
    """Only the last block can be partly filled, so waste is always < one block."""
    for L in range(1, 600):
        nb = oracle.blocks_needed(L, 16)
        assert (nb - 1) * 16 < L <= nb * 16
        assert 0 <= oracle.unused_slots(L, 16) < 16


def test_tiny_workload_block_count():
    """Tiny workload: lens {35,1,16,17} take 3+1+1+2 = 7 blocks of the 16-block pool."""
    w = wl.make("tiny")
    assert [len(t) for t in w.tables_host] == [3, 1, 1, 2]
    used = [b for t in w.tables_host for b in t]
    assert len(used) == 7 and len(set(used)) == 7
    assert all(0 <= b < 16 for b in used)
    assert w.num_blocks == 16


# ------------------------------------------------------------------ bf16 decode
def test_bf16_bits_widen_exactly():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x4049, 0x7F80], dtype=np.uint16)
    expect = [1.0, -2.0, 1.0078125, 0.0, -0.0, 3.140625, math.inf]
    # decode through the oracle: a one-token sequence returns its V row exactly
    D = len(bits)
    q = np.zeros((1, 1, D), np.uint16)
    kc = np.zeros((1, 1, 16, D), np.uint16)
    vc = np.zeros((1, 1, 16, D), np.uint16)
    vc[0, 0, 0, :] = bits
    vc[0, 0, 0, -1] = 0x3F80  # keep the row finite for the softmax
    out = oracle.paged_decode(q, kc, vc, np.zeros((1, 1), np.int32), np.array([1], np.int32), 1.0)
    assert list(out[0, 0, :-1]) == expect[:-1]
    assert out[0, 0, -1] == 1.0


# ------------------------------------------------------------------ cache write
def test_cache_write_matches_numpy_indexing():
    """Every written token is found at cache[slot // 16, h, slot % 16, :] (numpy's own
    indexing of the [NB][Hkv][B][D] layout), untouched slots keep their bytes, and
    negative slots write nothing."""
    rng = np.random.default_rng(0)
    NB, H, B, D, T = 9, 3, 16, 32, 20
    kc0 = rng.standard_normal((NB, H, B, D)).astype(np.float32)
    vc0 = rng.standard_normal((NB, H, B, D)).astype(np.float32)
    k = rng.standard_normal((T, H, D)).astype(np.float32)
    v = rng.standard_normal((T, H, D)).astype(np.float32)
    slots = rng.permutation(NB * B)[:T].astype(np.int64)
    slots[3] = -1
    slots[11] = -1
    kc, vc, bad = oracle.cache_write(k, v, slots, kc0, vc0)
    assert bad == 0
    touched = np.zeros((NB, B), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        touched[s // B, s % B] = True
        assert np.array_equal(kc[s // B, :, s % B, :], k[t])
        assert np.array_equal(vc[s // B, :, s % B, :], v[t])
    by_slot = lambda a: a.transpose(0, 2, 1, 3)  # [NB, B, H, D]
    assert np.array_equal(by_slot(kc)[~touched], by_slot(kc0)[~touched])
    assert np.array_equal(by_slot(vc)[~touched], by_slot(vc0)[~touched])


def test_cache_write_copies_bits_and_skips_out_of_range():
    NB, H, B, D = 2, 1, 16, 8
    kc0 = np.full((NB, H, B, D), 0xABCD, np.uint16)
    vc0 = np.full((NB, H, B, D), 0x1234, np.uint16)
    k = np.full((2, H, D), 0x7FC1, np.uint16)  # a NaN payload must travel unchanged
    v = np.full((2, H, D), 0xFFFF, np.uint16)
    kc, vc, bad = oracle.cache_write(k, v, np.array([17, NB * B], np.int64), kc0, vc0)
    assert bad == 1
    assert (kc[1, 0, 1] == 0x7FC1).all() and (vc[1, 0, 1] == 0xFFFF).all()
    kc[1, 0, 1] = 0xABCD
    vc[1, 0, 1] = 0x1234
    assert np.array_equal(kc, kc0) and np.array_equal(vc, vc0)


# ------------------------------------------------------------------ attention math
def _truth_pool(lens, Hq, Hkv, D, seed, bf16=False):
    """Contiguous per-sequence K/V written into a paged pool with the (pinned)
    cache write; returns (workload skeleton, truth lists, q, pools)."""
    rng = np.random.default_rng(seed)
    w = wl.build(lens, Hq, Hkv, D, torch.float32, seed=seed)
    NB = w.num_blocks
    kc = np.full((NB, Hkv, 16, D), np.nan, np.float32)
    vc = np.full((NB, Hkv, 16, D), np.nan, np.float32)
    if bf16:
        kc = np.full(kc.shape, 0x7FC0, np.uint16)
        vc = np.full(vc.shape, 0x7FC0, np.uint16)
    Ks, Vs = [], []
    for s, L in enumerate(lens):
        K = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        V = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        if bf16:
            K = torch.from_numpy(K).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            V = torch.from_numpy(V).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        slots = np.array([w.tables_host[s][t // 16] * 16 + t % 16 for t in range(L)], np.int64)
        kc, vc, bad = oracle.cache_write(K, V, slots, kc, vc)
        assert bad == 0
        Ks.append(K)
        Vs.append(V)
    q = rng.standard_normal((len(lens), Hq, D)).astype(np.float32)
    if bf16:
        q = torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return w, Ks, Vs, q, kc, vc


def _f64(a):
    return oracle.bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 1), (8, 2), (6, 3)])
def test_decode_equals_library_sdpa_fp64(Hq, Hkv, bf16):
    """Oracle == torch's scaled_dot_product_attention in fp64 on the contiguous
    K/V the pool was built from (GQA: query head i uses kv head i // (Hq/Hkv))."""
    lens = [35, 1, 16, 17, 48, 3]
    D = 32
    w, Ks, Vs, q, kc, vc = _truth_pool(lens, Hq, Hkv, D, seed=7, bf16=bf16)
    scale = 0.37
    out = oracle.paged_decode(q, kc, vc, wl.as_numpy(w.block_tables), np.array(lens, np.int32), scale)
    g = Hq // Hkv
    for s, L in enumerate(lens):
        K = torch.from_numpy(_f64(Ks[s])).permute(1, 0, 2).repeat_interleave(g, dim=0)  # [Hq, L, D]
        V = torch.from_numpy(_f64(Vs[s])).permute(1, 0, 2).repeat_interleave(g, dim=0)
        Q = torch.from_numpy(_f64(q[s]))[:, None, :]  # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], scale=scale)[0, :, 0]
        np.testing.assert_allclose(out[s], ref.numpy(), rtol=0, atol=1e-12)


def test_selected_rows_equal_full_output():
    w = wl.make("tiny")
    full = _decode(w)
    rows = [(0, 1), (3, 0), (1, 1), (0, 0)]
    sel = _decode(w, rows=rows)
    for i, (s, h) in enumerate(rows):
        assert np.array_equal(sel[i], full[s, h])


def test_single_token_returns_its_value_row():
    """L = 1: the softmax weight is exactly 1, so out = v_0."""
    w = wl.build([1, 1, 1], 4, 2, 64, torch.float32, seed=3)
    out = _decode(w)
    h = _np_host(w)
    for s in range(3):
        b = w.tables_host[s][0]
        for qh in range(4):
            assert np.array_equal(out[s, qh], h["vc"][b, qh // 2, 0].astype(np.float64))


def test_zero_query_gives_mean_of_values():
    """q = 0: all scores equal, so out = mean over the sequence of V."""
    w = wl.build([35, 17, 64], 2, 1, 32, torch.float32, seed=4)
    h = _np_host(w)
    h["q"][:] = 0
    out = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale)
    for s, L in enumerate(w.lens_host):
        rows = [h["vc"][w.tables_host[s][t // 16], 0, t % 16].astype(np.float64) for t in range(L)]
        np.testing.assert_allclose(out[s, 0], np.mean(rows, axis=0), rtol=0, atol=1e-13)


def test_two_tokens_closed_form():
    """Two tokens: out = sigma(z0 - z1) v0 + sigma(z1 - z0) v1 with z = scale q.k."""
    w = wl.build([2], 1, 1, 16, torch.float32, seed=5)
    h = _np_host(w)
    b = w.tables_host[0][0]
    qv = h["q"][0, 0].astype(np.float64)
    k0, k1 = h["kc"][b, 0, 0].astype(np.float64), h["kc"][b, 0, 1].astype(np.float64)
    v0, v1 = h["vc"][b, 0, 0].astype(np.float64), h["vc"][b, 0, 1].astype(np.float64)
    z0, z1 = w.scale * qv @ k0, w.scale * qv @ k1
    sig = 1.0 / (1.0 + math.exp(-(z0 - z1)))
    np.testing.assert_allclose(_decode(w)[0, 0], sig * v0 + (1 - sig) * v1, rtol=0, atol=1e-14)


def test_dominant_key_selects_its_value():
    """One key aligned with q and scaled far above the rest: out -> that token's V."""
    w = wl.build([40], 1, 1, 16, torch.float32, seed=6)
    h = _np_host(w)
    t_star = 21
    b = w.tables_host[0][t_star // 16]
    h["kc"][b, 0, t_star % 16] = 60.0 * h["q"][0, 0] / np.linalg.norm(h["q"][0, 0])
    out = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], 1.0)
    np.testing.assert_allclose(out[0, 0], h["vc"][b, 0, t_star % 16], rtol=0, atol=1e-9)


def test_zero_length_sequence_gives_zero_row():
    w = wl.build([0, 5], 2, 2, 16, torch.float32, seed=8)
    out = _decode(w)
    assert (out[0] == 0).all() and np.isfinite(out[1]).all()


# ------------------------------------------------------------------ paging invariances
def test_invariant_under_physical_permutation():
    """Moving blocks anywhere in the pool (tables updated) leaves the output unchanged."""
    w = wl.build([35, 1, 16, 17, 100], 4, 2, 32, torch.bfloat16, seed=9)
    h = _np_host(w)
    base = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale)
    perm = np.random.default_rng(1).permutation(w.num_blocks)  # new position of block b
    kc = np.empty_like(h["kc"])
    vc = np.empty_like(h["vc"])
    kc[perm] = h["kc"]
    vc[perm] = h["vc"]
    bt = np.where(h["bt"] >= 0, perm[np.maximum(h["bt"], 0)], -1).astype(np.int32)
    moved = oracle.paged_decode(h["q"], kc, vc, bt, h["sl"], w.scale)
    assert np.array_equal(base, moved)


@pytest.mark.parametrize("prefix_len", [64, 4090])
def test_shared_prefix_equals_private_copies(prefix_len):
    """Sequences pointing at shared prefix blocks give the same result as the same
    sequences holding private copies of those blocks."""
    lens = [prefix_len + s for s in (5, 40, 17)]
    w = wl.build(lens, 4, 2, 32, torch.bfloat16, seed=10, prefix_len=prefix_len)
    assert all(t[: prefix_len // 16] == w.tables_host[0][: prefix_len // 16] for t in w.tables_host)
    h = _np_host(w)
    shared = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale)
    # private copies: every sequence gets its own copy of every block it references
    refs = [b for t in w.tables_host for b in t]
    NB2 = len(refs)
    kc = np.zeros((NB2,) + h["kc"].shape[1:], h["kc"].dtype)
    vc = np.zeros_like(kc)
    bt = np.full_like(h["bt"], -1)
    i = 0
    for s, t in enumerate(w.tables_host):
        for j, b in enumerate(t):
            kc[i] = h["kc"][b]
            vc[i] = h["vc"][b]
            bt[s, j] = i
            i += 1
    private = oracle.paged_decode(h["q"], kc, vc, bt, h["sl"], w.scale)
    assert np.array_equal(shared, private)


def test_nan_in_unused_slots_does_not_leak():
    """Slots past each sequence's length (and unreferenced blocks) are never read."""
    clean = wl.build([35, 1, 16, 17, 50], 2, 1, 64, torch.float32, seed=11)
    dirty = wl.build([35, 1, 16, 17, 50], 2, 1, 64, torch.float32, seed=11, poison_unused=True)
    assert torch.isnan(dirty.k_cache).any()
    a, b = _decode(clean), _decode(dirty)
    assert np.isfinite(b).all() and np.array_equal(a, b)


# ------------------------------------------------------------------ split-K algebra
@pytest.mark.parametrize("partition_tokens", [16, 32, 48, 512])
def test_lse_merge_of_partitions_equals_unsplit(partition_tokens):
    w = wl.build([35, 1, 16, 17, 600, 513, 0], 4, 2, 32, torch.bfloat16, seed=12)
    h = _np_host(w)
    full = oracle.paged_decode(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale)
    m, l, acc, nparts = oracle.decode_partials(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, partition_tokens)
    assert list(nparts) == [-(-L // partition_tokens) for L in w.lens_host]
    merged = oracle.lse_merge(m, l, acc, nparts)
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-12)


def test_single_partition_is_the_unnormalised_softmax():
    """One partition: acc / l is the output and m is the largest score."""
    w = wl.build([30], 1, 1, 16, torch.float32, seed=13)
    h = _np_host(w)
    m, l, acc, nparts = oracle.decode_partials(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], w.scale, 512)
    out = _decode(w)
    np.testing.assert_allclose(acc[0, 0, 0] / l[0, 0, 0], out[0, 0], rtol=0, atol=1e-13)
    b = w.tables_host[0]
    scores = [w.scale * float(h["q"][0, 0].astype(np.float64) @ h["kc"][b[t // 16], 0, t % 16].astype(np.float64))
              for t in range(30)]
    assert m[0, 0, 0] == pytest.approx(max(scores), abs=1e-14)


# ------------------------------------------------------------------ block copy
def test_copy_blocks_matches_numpy_indexing():
    """dst blocks become byte copies of src blocks in both pools; others untouched;
    pairs outside the pool are skipped."""
    rng = np.random.default_rng(21)
    kc = rng.integers(0, 1 << 16, size=(9, 3, 16, 8), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(9, 3, 16, 8), dtype=np.uint16)
    src = np.array([1, 4, 7, 2], np.int32)
    dst = np.array([0, 5, 3, 9], np.int32)  # the last pair points outside the pool
    k2, v2, bad = oracle.copy_blocks(kc, vc, src, dst)
    assert bad == 1
    ek, ev = kc.copy(), vc.copy()
    ek[dst[:3]] = kc[src[:3]]
    ev[dst[:3]] = vc[src[:3]]
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)


# ------------------------------------------------------------------ several query tokens
def test_multi_query_with_one_token_each_is_decode():
    w = wl.build([35, 1, 16, 17, 90], 4, 2, 32, torch.bfloat16, seed=31)
    h = _np_host(w)
    qs = np.arange(w.num_seqs + 1, dtype=np.int32)
    multi = oracle.paged_decode_multi(h["q"], h["kc"], h["vc"], h["bt"], h["sl"], qs, w.scale)
    assert np.array_equal(multi, _decode(w))


def test_multi_query_token_equals_decode_of_the_truncated_sequence():
    """Query token r of n sees exactly the first L - n + r + 1 tokens."""
    lens = [40, 17, 70]
    nq = [3, 1, 5]
    w = wl.build(lens, 2, 1, 32, torch.float32, seed=32)
    h = _np_host(w)
    rng = np.random.default_rng(0)
    q = rng.standard_normal((sum(nq), 2, 32)).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    multi = oracle.paged_decode_multi(q, h["kc"], h["vc"], h["bt"], h["sl"], qs, w.scale)
    for s, (L, n) in enumerate(zip(lens, nq)):
        for r in range(n):
            row = qs[s] + r
            sl = np.array([L - n + r + 1], np.int32)
            one = oracle.paged_decode(q[row:row + 1], h["kc"], h["vc"], h["bt"][s:s + 1], sl, w.scale)
            assert np.array_equal(multi[row], one[0])


@pytest.mark.parametrize("Hq,Hkv", [(2, 1), (4, 2)])
def test_multi_query_equals_library_sdpa_with_causal_mask(Hq, Hkv):
    """Against torch SDPA in fp64 with an explicit mask on the contiguous K/V the
    pool was built from: new token r of n may see keys 0 .. L - n + r."""
    lens = [35, 18, 64]
    nq = [4, 2, 7]
    D = 32
    w, Ks, Vs, _, kc, vc = _truth_pool(lens, Hq, Hkv, D, seed=33)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((sum(nq), Hq, D)).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    out = oracle.paged_decode_multi(q, kc, vc, wl.as_numpy(w.block_tables), np.array(lens, np.int32), qs, 0.29)
    g = Hq // Hkv
    for s, (L, n) in enumerate(zip(lens, nq)):
        K = torch.from_numpy(Ks[s].astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, dim=0)
        V = torch.from_numpy(Vs[s].astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, dim=0)
        Q = torch.from_numpy(q[qs[s]:qs[s + 1]].astype(np.float64)).permute(1, 0, 2)  # [Hq, n, D]
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]     # [n, L]
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=mask,
                                                               scale=0.29)[0]
        np.testing.assert_allclose(out[qs[s]:qs[s + 1]], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ FP8 E4M3
@pytest.mark.parametrize("value,code", [
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE),
    (2.0 ** -9, 0x01), (2.0 ** -6, 0x08), (7 * 2.0 ** -9, 0x07), (1.125, 0x39), (240.0, 0x77),
    (2.0 ** -10, 0x00),            # half the smallest subnormal: tie, to even (zero)
    (3 * 2.0 ** -10, 0x02),        # 1.5 quanta: tie, to even (2)
    (1.0625, 0x38),                # halfway 1.0 / 1.125: to even (1.0)
    (1.1875, 0x3A),                # halfway 1.125 / 1.25: to even (1.25)
    (1.0626, 0x39),                # just above the tie
    (500.0, 0x7E), (1e30, 0x7E), (float("inf"), 0x7E), (-1e30, 0xFE),  # saturate at 448
])
def test_e4m3_known_codes(value, code):
    assert oracle.e4m3_encode(value) == code


def test_e4m3_nan_and_round_trip_of_every_code():
    assert oracle.e4m3_encode(float("nan")) == 0x7F
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    values = []
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        v = oracle.e4m3_decode(c)
        assert oracle.e4m3_encode(v) == c          # every finite code is its own nearest value
        values.append(v)
    pos = sorted(set(v for v in values if v > 0))
    assert len(pos) == 126 and pos[0] == 2.0 ** -9 and pos[-1] == 448.0
    # between neighbours, values round to the nearer one
    for a, b in zip(pos, pos[1:]):
        assert oracle.e4m3_decode(oracle.e4m3_encode(a + (b - a) * 0.49)) == a
        assert oracle.e4m3_decode(oracle.e4m3_encode(a + (b - a) * 0.51)) == b


def test_fp8_cache_write_quantises_and_places_codes():
    rng = np.random.default_rng(40)
    NB, H, B, D, T = 5, 2, 16, 16, 6
    k = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32)).to(torch.bfloat16)
    inv = np.array([40.0, 0.5], np.float32)
    slots = np.array([3, 17, -1, 40, 79, 0], np.int64)
    kc0 = np.full((NB, H, B, D), 0xAA, np.uint8)
    kc, vc, bad = oracle.cache_write_fp8(wl.as_numpy(k), wl.as_numpy(v), slots, kc0, kc0, inv, inv)
    assert bad == 0
    kf = k.float().numpy()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        for hh in range(H):
            want = [oracle.e4m3_encode(np.float32(x) * inv[hh]) for x in kf[t, hh]]
            assert list(kc[s // 16, hh, s % 16]) == want
    assert (kc[0, :, 1] == 0xAA).all()  # an untouched slot


def test_fp8_decode_reduces_to_the_bf16_oracle_on_representable_values():
    """Codes whose values (times a power-of-two scale) are exact in bf16 give the
    bf16 oracle's result."""
    w = wl.build([35, 1, 16, 70], 4, 2, 32, torch.bfloat16, seed=41)
    rng = np.random.default_rng(41)
    NB = w.num_blocks
    codes_k = rng.integers(0, 256, size=(NB, 2, 16, 32)).astype(np.uint8)
    codes_v = rng.integers(0, 256, size=(NB, 2, 16, 32)).astype(np.uint8)
    codes_k[(codes_k & 0x7F) == 0x7F] = 0x38   # no NaN codes
    codes_v[(codes_v & 0x7F) == 0x7F] = 0x38
    codes_k &= 0xBF  # keep magnitudes moderate (exponent field < 8)
    scales = np.array([0.25, 2.0], np.float32)
    dec = np.vectorize(oracle.e4m3_decode)
    kv = (dec(codes_k) * scales[None, :, None, None]).astype(np.float32)
    vv = (dec(codes_v) * scales[None, :, None, None]).astype(np.float32)
    kb = torch.from_numpy(kv).to(torch.bfloat16)
    vb = torch.from_numpy(vv).to(torch.bfloat16)
    assert torch.equal(kb.float(), torch.from_numpy(kv)) and torch.equal(vb.float(), torch.from_numpy(vv))
    h = _np_host(w)
    fp8 = oracle.paged_decode_fp8(h["q"], codes_k, codes_v, h["bt"], h["sl"], scales, scales, w.scale)
    bf = oracle.paged_decode(h["q"], wl.as_numpy(kb), wl.as_numpy(vb), h["bt"], h["sl"], w.scale)
    assert np.array_equal(fp8, bf)
