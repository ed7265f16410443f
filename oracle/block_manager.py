"""KV block manager: free list, reference counts, fork, copy-on-write
(oracle; test infrastructure).

What the pages fix:

* [P1] section 2: physical blocks are handed out one at a time, only as new
  tokens arrive; a block table maps logical to physical blocks.
* [P3] second paragraph: a KV cache manager keeps one block table per request,
  and blocks can be shared within and across a batch.
* [P1] section 3: parallel-sampling or beam-search branches all share the same
  physical prompt blocks; a branch that generates a token gets its own private
  block.

Policy where the pages are silent (the same policy is implemented by the
native manager, so the two are compared bit for bit):

* the free list is first-in-first-out: allocation takes from the front, a
  block whose reference count drops to zero goes to the back; it starts as the
  given ``free_order`` (default 0 .. n-1);
* ``allocate(seq, n)`` takes ceil(n / B) blocks at once for a prompt of n
  tokens and returns the n slots, slot = block * B + offset;
* ``append_slot(seq)`` adds one token at position t = len:
  if t % B == 0 a new block is taken; otherwise, if the last block is shared
  (reference count > 1), a new block is taken, the pair (last, new) is
  returned for a copy, the old block loses one reference and the table points
  at the new block (the last remaining holder then writes in place);
  otherwise the token goes into the last block;
* ``fork(parent, child)`` gives the child a copy of the parent's table and
  length and adds one reference to every block;
* ``free(seq)`` drops one reference from each block of the sequence;
* a failing call raises and leaves the state unchanged.

Prefix caching across requests ([P3] second paragraph: blocks may be shared
across the requests of a batch, not only within one; [P2] introduction and
"From Contiguous Reserves to Paged KV Blocks": block tables make KV memory
reusable and shareable).  The pages give no mechanism; the plainest reading,
taken here: a block that a prompt fills completely is identified by its
content, i.e. the whole token prefix up to the end of that block (the K/V of
a position depend on every token before it).

* ``allocate_prefix(seq, tokens)`` looks the prompt's full blocks up in
  order, prefix by prefix, and stops at the first one not cached; each hit
  joins the sequence's table with one more reference (a cached block whose
  count had dropped to zero leaves the free list).  The other blocks are
  taken from the front of the free list as in ``allocate``; every full one
  is then entered in the cache under its prefix (replacing any older entry
  for the same prefix).  Slots of tokens in hit blocks come back as -1: their
  K/V are already in the pool, and the cache write skips them.
* a freed block keeps its entry while it waits in the free list; it leaves
  the cache when the free list hands it out again (to any allocation).
* only prompt blocks are entered; blocks filled later by appends are not.
"""
from __future__ import annotations

from collections import deque


class NoBlocks(Exception):
    pass


class UnknownSeq(Exception):
    pass


class SeqExists(Exception):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad pool")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.cache: dict[tuple, int] = {}      # token prefix of a full block -> block
        self.key_of: dict[int, tuple] = {}     # block -> its prefix while cached

    # -- helpers ------------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        self.ref[b] = 1
        self._uncache(b)
        return b

    def _uncache(self, b: int) -> None:
        key = self.key_of.pop(b, None)
        if key is not None:
            del self.cache[key]

    def _slot(self, seq: int, t: int) -> int:
        B = self.block_size
        return self.tables[seq][t // B] * B + t % B

    # -- operations ---------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> list[int]:
        if seq in self.tables:
            raise SeqExists(seq)
        if num_tokens < 0:
            raise ValueError(num_tokens)
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise NoBlocks(need)
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = num_tokens
        return [self._slot(seq, t) for t in range(num_tokens)]

    def allocate_prefix(self, seq: int, tokens) -> tuple[list[int], int]:
        """Allocate a prompt reusing cached full blocks; returns (slots with
        -1 for cached tokens, number of cached tokens)."""
        if seq in self.tables:
            raise SeqExists(seq)
        tokens = [int(x) for x in tokens]
        B = self.block_size
        n = len(tokens)
        need = -(-n // B)
        full = n // B
        hits = []
        for j in range(full):
            b = self.cache.get(tuple(tokens[:(j + 1) * B]))
            if b is None:
                break
            hits.append(b)
        revived = sum(1 for b in hits if self.ref[b] == 0)
        if need - len(hits) > len(self.free) - revived:
            raise NoBlocks(need - len(hits))
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
        table = hits + [self._take() for _ in range(need - len(hits))]
        for j in range(len(hits), full):
            key = tuple(tokens[:(j + 1) * B])
            old = self.cache.get(key)
            if old is not None:
                del self.key_of[old]
            self.cache[key] = table[j]
            self.key_of[table[j]] = key
        self.tables[seq] = table
        self.lens[seq] = n
        cached = len(hits) * B
        return [-1 if t < cached else self._slot(seq, t) for t in range(n)], cached

    def num_cached(self) -> int:
        """Blocks currently entered in the prefix cache (held or free)."""
        return len(self.cache)

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables:
            raise UnknownSeq(parent)
        if child in self.tables:
            raise SeqExists(child)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append_slot(self, seq: int):
        """Returns (slot, cow) where cow is None or the (src, dst) block pair."""
        if seq not in self.tables:
            raise UnknownSeq(seq)
        B = self.block_size
        table = self.tables[seq]
        t = self.lens[seq]
        cow = None
        if t % B == 0:
            if not self.free:
                raise NoBlocks(1)
            table.append(self._take())
        elif self.ref[table[-1]] > 1:
            if not self.free:
                raise NoBlocks(1)
            old = table[-1]
            new = self._take()
            self.ref[old] -= 1
            table[-1] = new
            cow = (old, new)
        self.lens[seq] = t + 1
        return self._slot(seq, t), cow

    def free_seq(self, seq: int) -> None:
        if seq not in self.tables:
            raise UnknownSeq(seq)
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    # -- queries ------------------------------------------------------------
    def block_table(self, seq: int) -> list[int]:
        if seq not in self.tables:
            raise UnknownSeq(seq)
        return list(self.tables[seq])

    def seq_len(self, seq: int) -> int:
        if seq not in self.lens:
            raise UnknownSeq(seq)
        return self.lens[seq]

    def num_free(self) -> int:
        return len(self.free)

    def ref_count(self, block: int) -> int:
        return self.ref[block]

    def seqs(self):
        return sorted(self.tables)
