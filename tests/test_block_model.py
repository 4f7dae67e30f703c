"""Pins of the block-bookkeeping reference model against what the pages state."""
import json
import os

import pytest

from oracle.block_model import BlockModel, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example_35_tokens_takes_three_blocks():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_35_tokens.json")))
    m = BlockModel(8, g["block_size"])
    m.add(0)
    slots, copies = m.append(0, g["seq_len"])
    assert len(m.tables[0]) == g["blocks"] and copies == []
    assert len(m.tables[0]) * g["block_size"] - m.lens[0] == g["unused_slots"]
    assert m.num_free() == 8 - g["blocks"]
    # slots are the logical positions mapped through the table
    assert slots == [m.tables[0][p // 16] * 16 + p % 16 for p in range(35)]


def test_blocks_are_added_as_the_sequence_grows_and_freed_at_the_end():
    m = BlockModel(10)
    m.add(0)
    for L in range(1, 81):
        m.append(0, 1)
        assert len(m.tables[0]) == -(-L // 16)       # only the last block is partial
    assert m.num_free() == 10 - 5
    m.release(0)
    assert m.num_free() == 10 and all(r == 0 for r in m.ref)


def test_fork_shares_blocks_and_copies_only_on_divergence():
    m = BlockModel(16)
    m.add("prompt")
    m.append("prompt", 35)                            # blocks a, b, c(partial)
    a, b, c = m.tables["prompt"]
    for child in ("x", "y"):
        m.fork("prompt", child)
    assert m.ref[a] == m.ref[b] == m.ref[c] == 3
    sx, cx = m.append("x", 1)                          # x writes into the shared partial block
    assert len(cx) == 1 and cx[0][0] == c
    new_c = cx[0][1]
    assert m.tables["x"] == [a, b, new_c] and m.ref[c] == 2 and m.ref[new_c] == 1
    assert sx == [new_c * 16 + 35 % 16]
    sy, cy = m.append("y", 20)                         # y too: its own copy, then a new block
    assert len(cy) == 1 and cy[0][0] == c and m.ref[c] == 1
    assert len(m.tables["y"]) == 4
    # the prompt itself is the last holder of c: no copy when it writes
    sp, cp = m.append("prompt", 1)
    assert cp == [] and sp == [c * 16 + 3]


def test_full_shared_blocks_are_never_copied():
    m = BlockModel(8)
    m.add(0)
    m.append(0, 32)                                    # two full blocks
    m.fork(0, 1)
    s, c = m.append(1, 5)
    assert c == [] and len(m.tables[1]) == 3 and m.tables[1][:2] == m.tables[0]


def test_out_of_blocks_leaves_state_unchanged():
    m = BlockModel(2)
    m.add(0)
    m.append(0, 20)
    with pytest.raises(OutOfBlocks):
        m.append(0, 20)
    assert m.lens[0] == 20 and len(m.tables[0]) == 2
