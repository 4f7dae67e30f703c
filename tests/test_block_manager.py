"""The library's native block manager (host code, no GPU) against the reference
model, operation by operation, plus the pages' allocation rules through the
native API."""
import json
import os
import random

import pytest

from oracle.block_model import BlockModel, OutOfBlocks
from paged_kv_cache_432_b200 import build as pa_build
from paged_kv_cache_432_b200 import pagedattn as pa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pa_build.build()


def _same_state(bm, model, nb):
    assert bm.num_free() == model.num_free()
    for b in range(nb):
        assert bm.refcount(b) == model.ref[b], b
    ids = sorted(model.tables)
    if ids:
        width = max(1, max(len(t) for t in model.tables.values()))
        tab, lens = bm.tables(ids, width)
        for i, s in enumerate(ids):
            t = model.tables[s]
            assert tab[i, : len(t)].tolist() == t and (tab[i, len(t):] == -1).all()
            assert int(lens[i]) == model.lens[s]


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_the_model(seed):
    rng = random.Random(seed)
    NB = 48
    bm, model = pa.BlockManager(NB, 16), BlockModel(NB, 16)
    live, next_id = [], 0
    for step in range(400):
        op = rng.random()
        if not live or op < 0.15:
            bm.add(next_id)
            model.add(next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.3:
            parent = rng.choice(live)
            bm.fork(parent, next_id)
            model.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.85:
            s, n = rng.choice(live), rng.choice([1, 1, 1, 3, 16, 17, 40])
            try:
                want = model.append(s, n)
            except OutOfBlocks:
                with pytest.raises(pa.PagedAttnError) as e:
                    bm.append(s, n)
                assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS
            else:
                assert bm.append(s, n) == want
        else:
            s = live.pop(rng.randrange(len(live)))
            bm.release(s)
            model.release(s)
        if step % 25 == 0:
            _same_state(bm, model, NB)
    _same_state(bm, model, NB)


def test_worked_example_through_the_native_manager():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_35_tokens.json")))
    bm = pa.BlockManager(8, g["block_size"])
    bm.add(0)
    slots, copies = bm.append(0, g["seq_len"])
    tab, lens = bm.tables([0], 4)
    assert (tab[0] >= 0).sum() == g["blocks"] and copies == [] and int(lens[0]) == 35
    assert bm.num_free() == 8 - g["blocks"]
    assert slots[-1] % 16 == (35 - 1) % 16


def test_copy_on_write_and_errors():
    bm = pa.BlockManager(6, 16, max_blocks_per_seq=3)
    bm.add(0)
    bm.append(0, 20)                       # blocks a, b(partial)
    bm.fork(0, 1)
    (tab, _) = bm.tables([0, 1], 3)
    a, b = tab[0, :2].tolist()
    assert bm.refcount(a) == bm.refcount(b) == 2
    slots, copies = bm.append(1, 1)        # writes into shared partial b -> copied
    assert copies[0][0] == b and bm.refcount(b) == 1
    nb = copies[0][1]
    assert slots == [nb * 16 + 4]
    with pytest.raises(pa.PagedAttnError):
        bm.add(0)                          # id in use
    with pytest.raises(pa.PagedAttnError):
        bm.append(7, 1)                    # unknown sequence
    with pytest.raises(pa.PagedAttnError):
        bm.append(0, 40)                   # beyond max_blocks_per_seq
    bm.release(0)
    bm.release(1)
    assert bm.num_free() == 6
