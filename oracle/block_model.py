"""Reference model of paged KV-block bookkeeping (plain Python).

TEST INFRASTRUCTURE, like the rest of this package: the library's native
block manager is checked against this model operation by operation.

What it follows: "Was ändert PagedAttention an der KV-Speicherzuweisung für
LLMs?" (slavadubrov.com), §"Ungenutzten Platz in Blöcken berechnen" (fixed
16-token blocks, only the last one partly filled; blocks are added as a
sequence grows and released when its request ends) and §"Gemeinsame Nutzung
erfordert mehr als Speicherzuweisung" (several requests may reference one
block; copy-on-write lets them diverge without corrupting the shared state);
"PagedAttention et vLLM" (aiunderstanding.org), §"Questions fréquemment
posées" (sequences with identical prefixes point at the same physical pages
and copy only when a branch diverges).

Rules, written out:
  * free blocks are handed out first-in first-out from a free list that starts
    in ascending id order;
  * a sequence holds ceil(len / B) blocks; appending n tokens fills the last
    block first and takes new blocks from the free list as needed;
  * fork(parent, child): the child gets the parent's table and length; every
    block's reference count goes up by one;
  * before a sequence writes into its last block, if that block is partly
    filled and shared (reference count > 1), the sequence gets a fresh block,
    a copy (old -> new) is recorded for the device, and the old block's count
    goes down (copy-on-write); full shared blocks are never written again;
  * free(seq): every block's count goes down; blocks at zero return to the
    end of the free list.
"""
from collections import deque


class OutOfBlocks(Exception):
    pass


class BlockModel:
    def __init__(self, num_blocks: int, block_size: int = 16):
        self.B = block_size
        self.free = deque(range(num_blocks))
        self.ref = [0] * num_blocks
        self.tables = {}
        self.lens = {}

    def add(self, seq):
        assert seq not in self.tables
        self.tables[seq] = []
        self.lens[seq] = 0

    def fork(self, parent, child):
        assert child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def _take(self):
        if not self.free:
            raise OutOfBlocks()
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def append(self, seq, n):
        """Reserve n token slots at the end of seq; returns (slots, copies)."""
        t, L, B = self.tables[seq], self.lens[seq], self.B
        # blocks needed beyond the current ones, plus a possible copy
        new_blocks = -(-(L + n) // B) - len(t)
        cow = n > 0 and L % B != 0 and self.ref[t[-1]] > 1
        if new_blocks + (1 if cow else 0) > len(self.free):
            raise OutOfBlocks()
        copies = []
        if cow:
            old = t[-1]
            nb = self._take()
            copies.append((old, nb))
            self.ref[old] -= 1
            t[-1] = nb
        slots = []
        for pos in range(L, L + n):
            if pos // B == len(t):
                t.append(self._take())
            slots.append(t[pos // B] * B + pos % B)
        self.lens[seq] = L + n
        return slots, copies

    def release(self, seq):
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    def num_free(self):
        return len(self.free)
