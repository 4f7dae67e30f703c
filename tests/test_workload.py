"""The seeded generator builds the five workloads with the stated structure."""
import math

import pytest
import torch

from paged_kv_cache_432_b200 import workload as wl


@pytest.mark.parametrize("name", ["tiny", "mha", "gqa", "prefix", "long"])
def test_plan_structure(name):
    p = wl.config_plan(name, seed=0)
    nb = [len(t) for t in p.tables]
    assert nb == [-(-L // 16) for L in p.lens]
    ids = [b for t in p.tables for b in t]
    assert all(0 <= b < p.num_blocks for b in ids)
    if name == "prefix":
        # every table starts with the same 256 shared blocks; everything else is private
        assert all(t[:256] == p.tables[0][:256] for t in p.tables)
        private = [b for t in p.tables for b in t[256:]]
        assert len(set(private)) == len(private)
        assert not set(private) & set(p.tables[0][:256])
    else:
        assert len(set(ids)) == len(ids), "a block is owned by one sequence"
    if name == "tiny":
        assert p.num_blocks == 16
    else:
        assert p.num_blocks == math.ceil(1.25 * p.needed_blocks)


def test_length_distributions():
    mha = wl.config_plan("mha").lens
    assert len(mha) == 64 and min(mha) >= 128 and max(mha) <= 2048
    gqa = wl.config_plan("gqa").lens
    assert len(gqa) == 256 and min(gqa) >= 16 and max(gqa) <= 8192
    med = sorted(gqa)[128]
    assert 700 < med < 1500  # lognormal with median 1024
    pre = wl.config_plan("prefix").lens
    assert len(pre) == 128 and all(4096 + 64 <= L <= 4096 + 512 for L in pre)
    lo = wl.config_plan("long").lens
    assert len(lo) == 8 and all(32768 <= L <= 131072 for L in lo)


def test_seeded_and_distinct():
    assert wl.config_plan("gqa", 0).tables == wl.config_plan("gqa", 0).tables
    assert wl.config_plan("gqa", 0).lens != wl.config_plan("gqa", 1).lens


def test_new_token_slot_is_last_position():
    w = wl.build([35, 1, 16, 17, 0], 2, 1, 16, torch.float32, seed=2)
    for s, L in enumerate(w.lens_host):
        slot = int(w.slot_mapping[s])
        if L == 0:
            assert slot == -1
            continue
        assert slot // 16 == w.tables_host[s][(L - 1) // 16]
        assert slot % 16 == (L - 1) % 16


def test_copy_on_write_of_partial_prefix_block():
    """A prefix ending mid-block: each sequence's first private block starts with a
    copy of the shared partial block's tokens."""
    w = wl.build([4090 + 5, 4090 + 40], 2, 1, 16, torch.bfloat16, seed=3, prefix_len=4090)
    p = wl.plan(w.lens_host, seed=3, prefix_len=4090)
    assert len(p.cow_pairs) == 2
    for src, dst, rem in p.cow_pairs:
        assert rem == 10
        assert torch.equal(w.k_cache[dst, :, :10], w.k_cache[src, :, :10])
        assert not torch.equal(w.k_cache[dst, :, 10:], w.k_cache[src, :, 10:])
    # the copies are private: different tables, same logical prefix
    assert w.tables_host[0][255] != w.tables_host[1][255]
    assert w.tables_host[0][:255] == w.tables_host[1][:255]


def test_poison_marks_only_unreachable_slots():
    w = wl.build([35, 1], 2, 1, 16, torch.float32, seed=4, poison_unused=True)
    nan = torch.isnan(w.k_cache[:, 0, :, 0])
    for s, L in enumerate(w.lens_host):
        for t in range(L):
            assert not nan[w.tables_host[s][t // 16], t % 16]
    assert int(nan.sum()) == w.num_blocks * 16 - sum(w.lens_host)


def test_fp8_pools_draw_no_nan_code_and_poison_only_unreachable_slots():
    w = wl.build([35, 1, 300], 4, 2, 64, torch.bfloat16, seed=6)
    kc, vc, ks, vs = wl.fp8_pools(w)
    for c in (kc, vc):
        assert c.dtype == torch.uint8 and c.shape == (w.num_blocks, 2, 16, 64)
        assert not bool(((c & 0x7F) == 0x7F).any())  # neither NaN code is drawn
        assert int(c.unique().numel()) > 200          # the other codes all appear
    assert ks.shape == (2,) and bool(((ks >= 1 / 160) & (ks <= 1 / 112)).all())
    kc2, _, ks2, _ = wl.fp8_pools(w)
    assert torch.equal(kc, kc2) and torch.equal(ks, ks2)  # seeded
    assert not torch.equal(kc, wl.fp8_pools(w, seed=9)[0])
    kp, _, _, _ = wl.fp8_pools(w, poison_unused=True)
    nan = kp[:, 0, :, 0] == wl.E4M3_NAN
    for s, L in enumerate(w.lens_host):
        for t in range(L):
            assert not nan[w.tables_host[s][t // 16], t % 16]
    assert int(nan.sum()) == w.num_blocks * 16 - sum(w.lens_host)


def test_prompt_groups_share_their_own_prefix_blocks():
    """Several prompt groups: the tables of a group start with the same full
    blocks (its own prompt), different groups share nothing, and a prompt
    ending mid-block gives each sequence of its group a private copy."""
    groups = [(3, 64), (2, 0), (4, 37)]
    lens = [64 + 5, 64 + 40, 64 + 16, 9, 300, 37 + 1, 37 + 20, 37 + 100, 37]
    w = wl.build(lens, 4, 2, 16, torch.bfloat16, seed=8, groups=groups)
    assert w.group_start_host == [0, 3, 5, 9] and w.group_blocks_host == [4, 0, 2]
    assert w.group_start.tolist() == [0, 3, 5, 9] and w.group_blocks.tolist() == [4, 0, 2]
    assert w.shared_prefix_blocks == 0
    t = w.tables_host
    assert t[0][:4] == t[1][:4] == t[2][:4]
    assert t[5][:2] == t[6][:2] == t[7][:2] == t[8][:2]
    assert t[5][2] != t[6][2]                     # the partial third block: private copies
    assert not set(t[0][:4]) & set(t[5][:2])      # the groups share nothing
    assert not set(t[3]) & set(t[4])
    p = wl.plan(lens, seed=8, groups=groups)
    assert sorted(rem for _, _, rem in p.cow_pairs) == [5] * 4
    for src, dst, rem in p.cow_pairs:
        assert torch.equal(w.k_cache[dst, :, :rem], w.k_cache[src, :, :rem])
    # one group of every sequence gives the same tables as the single-prefix form
    a = wl.plan(lens[:3], seed=2, prefix_len=64)
    b = wl.plan(lens[:3], seed=2, groups=[(3, 64)])
    assert a.tables == b.tables and a.num_blocks == b.num_blocks
